// Non-causal softmax attention over all latent tokens of a batch item, per
// head, on sm_100a tensor cores (bf16 operands, fp32 accumulation):
//   O[i] = sum_j softmax_j(Q[i].K[j] / sqrt(head_dim)) V[j]
// Q, K, V come head-major ([part][batch][head][token][lane], as the QKV
// projection writes them); O is written token-major ([batch][token][d]) in bf16
// together with each token's max |O| over all heads (the per-row scale of the
// quantizer ahead of the output projection).
//
// Method references (web pages on the h3.c / h3-metal engine):
//   "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론", section
//     "Metal 4 및 TensorOps": head-major Q/K/V as the attention input.
//   "맥북에서 AI 영상 생성 모델 돌리기 - MiniMax H3 로컬 실행과 30초 애니메이션 만들기",
//     section "★ 긴 영상은 나눠 찍는 게 훨씬 쌉니다": cost grows about as
//     frames^1.9, i.e. full attention over every latent token.
//
// Design (B200). One CTA per (256 queries, batch item x head): two query tiles
// g = 0, 1 of 128 rows share every K/V tile.
//   warp 0     TMA: Q0 and Q1 once, then K_j and V_j (128 keys) into 2-stage rings
//   warp 1     tcgen05.mma from one thread, in the order
//                S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) S0(2) ...
//              so the tensor core always has the other tile's work queued
//   warps 2-3  idle (they complete warpgroup 0 for the register split)
//   warps 4-7  softmax of tile 0, warps 8-11 softmax of tile 1 (thread = row)
// Registers: launched at 168 per thread (384 threads), warpgroup 0 gives up all
// but 56 (setmaxnreg.dec) and the two softmax warpgroups take 224 (setmaxnreg.inc),
// so that a thread's 128 scores, the exponential pipeline and the O rescale fit
// without spilling.
// Tensor memory (512 columns): S0 | S1 | O0 | O1. Each softmax thread reads its
// row of S_g, writes P_g = exp2(S*c - m) as bf16 pairs over the first 64
// columns of S_g, and the P V product takes its A operand from tensor memory.
// A commit tracks every earlier MMA of the issuing thread, so when S_g(j) is
// complete, PV_g(j-1) is complete too: O_g can be rescaled then without another
// barrier. The running max is kept until a row's max grows by more than 2^8
// (then O_g and the row sum are rescaled); the final division by the row sum
// is exact either way. Every wait is bounded and every decision guarding a
// warp-collective TMEM access is warp-uniform.
#include "h3b_common.cuh"
#include "h3b_internal.h"


namespace h3b {
namespace attn {
constexpr int BQ = 128, BKV = 128, kThreads = 384;
// registers per thread after the split: warpgroup 0 (TMA, MMA, two idle warps) gives
// up registers, the two softmax warpgroups take them (launch: 384 x 168 = 64512;
// 128 x 56 + 256 x 224 = 64512; per sub-partition 56 + 224 + 224 <= 512)
constexpr uint32_t kRegsControl = 56, kRegsSoftmax = 224;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BOX = 16384;  // one TMA box: 128 rows x 128 bytes
}  // namespace attn

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe, two lanes at a time: x = n + f with n = round(x) and
// f in [-1/2, 1/2]; 2^f by a cubic fitted here for minimax relative error on
// that interval (Remez exchange; max relative error 7.5e-5, below the 2^-9 of
// the bf16 rounding that P then goes through), and 2^n added to the exponent
// field. Adding 1.5 * 2^23 rounds x to an integer held in the low mantissa
// bits; x is clamped at -125 so that 2^n stays a normal number.
constexpr float kExp2C0 = 0.99992806f, kExp2C1 = 0.69326097f, kExp2C2 = 0.24261113f, kExp2C3 = 0.05517167f;
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
  const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
  const float2 r = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(r, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// tcgen05.mma with the A operand in tensor memory (kind::f16, bf16 inputs).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int DH>
struct AttnLayout {
  static constexpr int NBOX = DH / 64;             // TMA boxes per Q/K/V tile
  static constexpr int TILE = attn::BKV * DH * 2;  // bytes of one Q/K/V tile
  static constexpr int Q_OFF = 0;                  // Q0, Q1
  static constexpr int K_OFF = Q_OFF + 2 * TILE;   // K stages 0, 1
  static constexpr int V_OFF = K_OFF + 2 * TILE;   // V stages 0, 1
  static constexpr int BAR_OFF = V_OFF + 2 * TILE;
  static constexpr int NBARS = 16;
  static constexpr size_t SMEM_NEED = (size_t)BAR_OFF + NBARS * 8 + 16 + 1024;
  // At least 120 KB so two CTAs never share an SM: each holds all 512 TMEM columns.
  static constexpr size_t SMEM = SMEM_NEED > 120 * 1024 ? SMEM_NEED : 120 * 1024;
  // tensor memory columns: S0, S1, O0, O1
  static constexpr uint32_t S_COL0 = 0, S_COL1 = 128, O_COL0 = 256, O_COL1 = 256 + DH;
};

// kPolyMod: every kPolyMod-th pair of exponentials goes to the FMA pipe (0: none).
template <int DH, int kPolyMod>
__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a, float scale_log2) {
  using namespace attn;
  using Lay = AttnLayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb0 = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (3 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (5 + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (7 + s); };
  auto s_full = [&](int g) { return bar0 + 8u * (9 + g); };
  auto p_full = [&](int g) { return bar0 + 8u * (11 + g); };
  auto fin = [&](int g) { return bar0 + 8u * (13 + g); };
  const uint32_t drain = bar0 + 8u * 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Lay::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int BH = a.B * a.n_heads;
  const int L = a.L;
  const int nkv = (L + BKV - 1) / BKV;
  constexpr uint32_t IDESC_S = instr_desc(1, 1, 0, 0, BQ, BKV);
  constexpr uint32_t IDESC_PV = instr_desc(1, 1, 0, 1, BQ, DH);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(k_full(s), 1); mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1); mbar_init(v_empty(s), 1);
      mbar_init(s_full(s), 1); mbar_init(p_full(s), 4); mbar_init(fin(s), 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // Q, K, V are the previous grid's output
  griddep_launch_dependents();

  // each role changes its register budget at its start (all four warps of a warpgroup)
  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (lane == 0) {
      // ---------------- TMA producer
      bool ok = true;
      uint32_t filled = 0, fill_ph = 0;  // bits s (K stage s) and 2+s (V stage s)
      mbar_arrive_expect_tx(q_full, 2 * Lay::TILE);
      for (int g = 0; g < 2; ++g)
        for (int b = 0; b < Lay::NBOX; ++b)
          tma_load_3d(sb0 + Lay::Q_OFF + g * Lay::TILE + b * BOX, &tm, q_full, b * 64, qt * 2 * BQ + g * BQ, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait_or_abort(k_empty(s), ph ^ 1u, abort_flag, a.err, ERR_WAIT_MMA)) { ok = false; break; }
        mbar_arrive_expect_tx(k_full(s), Lay::TILE);
        for (int b = 0; b < Lay::NBOX; ++b)
          tma_load_3d(sb0 + Lay::K_OFF + s * Lay::TILE + b * BOX, &tm, k_full(s), b * 64, j * BKV, BH + bh);
        filled |= 1u << s;
        fill_ph = (fill_ph & ~(1u << s)) | (ph << s);
        if (!mbar_wait_or_abort(v_empty(s), ph ^ 1u, abort_flag, a.err, ERR_WAIT_MMA)) { ok = false; break; }
        mbar_arrive_expect_tx(v_full(s), Lay::TILE);
        for (int b = 0; b < Lay::NBOX; ++b)
          tma_load_3d(sb0 + Lay::V_OFF + s * Lay::TILE + b * BOX, &tm, v_full(s), b * 64, j * BKV, 2 * BH + bh);
        filled |= 4u << s;
        fill_ph = (fill_ph & ~(4u << s)) | (ph << (2 + s));
      }
      if (!ok) {
        *abort_flag = 1;
        mbar_wait(q_full, 0, a.err, ERR_WAIT_DRAIN, kDrainLimitNs);
        for (int s = 0; s < 2; ++s) {
          if (filled & (1u << s)) mbar_wait(k_full(s), (fill_ph >> s) & 1u, a.err, ERR_WAIT_DRAIN, kDrainLimitNs);
          if (filled & (4u << s)) mbar_wait(v_full(s), (fill_ph >> (2 + s)) & 1u, a.err, ERR_WAIT_DRAIN, kDrainLimitNs);
        }
      } else {
        for (int s = 0; s < 2; ++s) {  // tail: every issued tile has been consumed
          if (filled & (1u << s)) mbar_wait(k_empty(s), (fill_ph >> s) & 1u, a.err, ERR_WAIT_MMA);
          if (filled & (4u << s)) mbar_wait(v_empty(s), (fill_ph >> (2 + s)) & 1u, a.err, ERR_WAIT_MMA);
        }
      }
    }
  } else if (warp == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (lane == 0) {
      // ---------------- MMA issuer
      bool any = false;
      auto issue_s = [&](int g, int j) -> bool {  // S_g(j) = Q_g K_j^T
        const int s = j & 1;
        if (g == 0 && !mbar_wait_or_abort(k_full(s), (j >> 1) & 1, abort_flag, a.err, ERR_WAIT_TMA)) return false;
        tc_fence_after();
        const uint32_t q_addr = sb0 + Lay::Q_OFF + g * Lay::TILE;
        const uint32_t k_addr = sb0 + Lay::K_OFF + s * Lay::TILE;
        const uint32_t s_col = g == 0 ? Lay::S_COL0 : Lay::S_COL1;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(q_addr + (k >> 2) * BOX + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + (k >> 2) * BOX + (k & 3) * 32, 16, 1024);
          mma_f16(tmem + s_col, ad, bd, IDESC_S, k > 0 ? 1u : 0u);
        }
        any = true;
        tc_commit(s_full(g));
        if (g == 1) tc_commit(k_empty(s));
        return true;
      };
      auto issue_pv = [&](int g, int j) -> bool {  // O_g += P_g(j) V_j
        const int s = j & 1;
        if (!mbar_wait_or_abort(p_full(g), j & 1, abort_flag, a.err, ERR_WAIT_EPI)) return false;
        if (g == 0 && !mbar_wait_or_abort(v_full(s), (j >> 1) & 1, abort_flag, a.err, ERR_WAIT_TMA)) return false;
        tc_fence_after();
        const uint32_t v_addr = sb0 + Lay::V_OFF + s * Lay::TILE;
        const uint32_t o_col = g == 0 ? Lay::O_COL0 : Lay::O_COL1;
        const uint32_t s_col = g == 0 ? Lay::S_COL0 : Lay::S_COL1;
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint64_t bd = smem_desc_sw128(v_addr + k * 2048, BOX, 1024);
          mma_f16_ts(tmem + o_col, tmem + s_col + k * 8, bd, IDESC_PV, (j > 0 || k > 0) ? 1u : 0u);
        }
        if (g == 1) tc_commit(v_empty(s));
        return true;
      };
      bool ok = mbar_wait(q_full, 0, a.err, ERR_WAIT_TMA);
      ok = ok && issue_s(0, 0) && issue_s(1, 0);
      for (int j = 0; j < nkv && ok; ++j) {
        ok = issue_pv(0, j);
        if (!ok) break;
        if (j + 1 < nkv) ok = issue_s(0, j + 1);
        else tc_commit(fin(0));
        if (!ok) break;
        ok = issue_pv(1, j);
        if (!ok) break;
        if (j + 1 < nkv) ok = issue_s(1, j + 1);
        else tc_commit(fin(1));
      }
      if (!ok) {
        *abort_flag = 1;
        if (any) {
          tc_commit(drain);
          mbar_wait(drain, 0, a.err, ERR_WAIT_DRAIN, kDrainLimitNs);
        }
      }
    }
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ---------------- softmax warps: 4-7 -> tile 0, 8-11 -> tile 1 (thread = query row)
    const int g = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_lane = (uint32_t)(quad * 32) << 16;
    const uint32_t s_col = g == 0 ? Lay::S_COL0 : Lay::S_COL1;
    const uint32_t o_col = g == 0 ? Lay::O_COL0 : Lay::O_COL1;
    const float2 c2 = make_float2(scale_log2, scale_log2);
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const bool s_ok = mbar_wait_or_abort(s_full(g), j & 1, abort_flag, a.err, ERR_WAIT_MMA);
      if (!__all_sync(0xFFFFFFFFu, s_ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c)
        tmem_ld32(tmem + t_lane + s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) tmem_reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));

      const int nvalid = min(BKV, L - j * BKV);
      if (nvalid < BKV) {  // uniform: only the last, partial key tile
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (i >= nvalid) sr[i] = __float_as_uint(-INFINITY);
      }
      // row max with 8 independent partial maxima
      float pm[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) pm[t] = __uint_as_float(sr[t]);
#pragma unroll
      for (int i = 8; i < BKV; i += 16)
#pragma unroll
        for (int t = 0; t < 8; ++t) pm[t] = max3f(pm[t], __uint_as_float(sr[i + t]), __uint_as_float(sr[i + 8 + t]));
      const float mx = fmaxf(max3f(pm[0], pm[1], pm[2]), max3f(max3f(pm[3], pm[4], pm[5]), pm[6], pm[7]));
      const float mxs = mx * scale_log2;
      float alpha = 1.0f;
      bool rescale = false;
      if (j == 0) {
        m_run = mxs;
      } else if (mxs > m_run + 8.0f) {
        alpha = fast_exp2(m_run - mxs);
        m_run = mxs;
        rescale = true;
      }
      // p = exp2(s * c - m), packed to bf16 pairs in place; sum with 4 packed accumulators
      const float2 nm2 = make_float2(-m_run, -m_run);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int i = 0; i < BKV; i += 2) {
        const float2 t = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), c2, nm2);
        float2 p;
        if (kPolyMod > 0 && (i >> 1) % (kPolyMod > 0 ? kPolyMod : 1) == kPolyMod - 1)
          p = exp2_poly2(t);
        else
          p = make_float2(fast_exp2(t.x), fast_exp2(t.y));
        acc[(i >> 1) & 3] = __fadd2_rn(acc[(i >> 1) & 3], p);
        sr[i >> 1] = pack_bf16x2(p.x, p.y);
      }
      const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
      const float2 a03 = __fadd2_rn(a01, a23);
      l_run = fmaf(l_run, alpha, a03.x + a03.y);

      // S_g(j) complete => PV_g(j-1) complete: O_g is stable until P_g(j) is published.
      if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + t_lane + o_col + c * 32, o);
          tmem_ld_wait();
          tmem_reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                                        make_float2(alpha, alpha));
            o[e] = __float_as_uint(v.x);
            o[e + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tmem + t_lane + o_col + c * 32, o);
        }
      }
      // P_g(j) over the first 64 columns of S_g: column c holds keys 2c (low half) and 2c+1.
      tmem_st32(tmem + t_lane + s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_st32(tmem + t_lane + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(g));
    }
    const bool f_ok = ok && mbar_wait_or_abort(fin(g), 0, abort_flag, a.err, ERR_WAIT_MMA);
    if (__all_sync(0xFFFFFFFFu, f_ok)) {
      tc_fence_after();
      const int q = qt * 2 * BQ + g * BQ + row;
      const int b = bh / a.n_heads, h = bh - b * a.n_heads;
      const float inv_l = 1.0f / l_run;
      const float2 il2 = make_float2(inv_l, inv_l);
      float amax = 0.0f;
      const int dm = a.n_heads * DH;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.o) + ((size_t)b * L + q) * dm + h * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + t_lane + o_col + c * 32, o);
        tmem_ld_wait();
        tmem_reg_fence(o);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), il2);
          pk[e] = pack_bf16x2(v.x, v.y);
          amax = max3f(amax, fabsf(bf16_lo(pk[e])), fabsf(bf16_hi(pk[e])));
        }
        if (q < L && H3B_IDX_OK(((long long)b * L + q) * dm + h * DH + c * 32 + 31, (long long)a.B * L * dm, a.err)) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) d4[gg] = make_uint4(pk[4 * gg], pk[4 * gg + 1], pk[4 * gg + 2], pk[4 * gg + 3]);
        }
      }
      if (q < L && H3B_IDX_OK((long long)b * L + q, (long long)a.B * L, a.err))
        atomicMax(reinterpret_cast<unsigned*>(a.absmax) + (size_t)b * L + q, __float_as_uint(amax));
    } else {
      *abort_flag = 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int DH, int kPolyMod>
static cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  using Lay = AttnLayout<DH>;
  CUtensorMap tm;
  // qkv viewed as [3*B*H][L][DH]
  if (!make_tmap_3d(&tm, a.qkv, 2, (uint64_t)DH, (uint64_t)a.L, (uint64_t)3 * a.B * a.n_heads, 64, attn::BKV))
    return cudaErrorInvalidValue;
  auto k = attention_kernel<DH, kPolyMod>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.L + 2 * attn::BQ - 1) / (2 * attn::BQ), a.B * a.n_heads);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  return launch_pdl(k, grid, dim3(attn::kThreads), Lay::SMEM, st, tm, a, scale_log2);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.L == 0 || a.B == 0) return cudaSuccess;
  // One exponential pair in four on the FMA pipe: the measured best split between
  // the MUFU and FMA pipes at head_dim 128 (none: 0.59, one in two: 0.58,
  // one in four: 0.61 of the bf16 tensor peak at d = 5120, 18432 tokens).
  if (a.head_dim == 128) return launch_attn<128, 4>(a, st);
  if (a.head_dim == 64) return launch_attn<64, 4>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace h3b
