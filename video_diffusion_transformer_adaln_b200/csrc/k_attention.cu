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
// Design (B200): one CTA per (128-query tile, batch item x head). Warp 0 loads
// Q once and streams K/V tiles of 128 keys with TMA (2-stage rings, 128-byte
// swizzle); warp 1 issues tcgen05.mma from one thread: S = Q K^T into one of
// two TMEM score buffers, then O += P V into a TMEM accumulator, with the next
// tile's S issued ahead of the current P V. Warps 2-5 (one query row per
// thread) read S from TMEM, run the online softmax in fp32 with exp2, write P
// as bf16 into shared memory in the MMA operand layout, and rescale O in TMEM
// only when a row's running max grows by more than 2^8 (otherwise the stale
// max is kept; the final division by the row sum is exact either way).
#include "h3b_common.cuh"
#include "h3b_internal.h"

namespace h3b {
namespace attn {
constexpr int BQ = 128, BKV = 128, kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BOX = 16384;  // one TMA box: 128 rows x 128 bytes
}  // namespace attn

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int DH>
struct AttnLayout {
  static constexpr int NBOX = DH / 64;                // TMA boxes per Q/K/V tile
  static constexpr int TILE = attn::BKV * DH * 2;     // bytes of one Q/K/V tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + 2 * TILE;
  static constexpr int P_OFF = V_OFF + 2 * TILE;
  static constexpr int BAR_OFF = P_OFF + attn::BQ * attn::BKV * 2;
  static constexpr int NBARS = 1 + 8 + 2 + 2 + 1 + 1 + 1;
  // At least 120 KB so that two CTAs never share an SM: each holds all 512
  // TMEM columns for its lifetime.
  static constexpr size_t SMEM_NEED = (size_t)BAR_OFF + NBARS * 8 + 16 + 1024;
  static constexpr size_t SMEM = SMEM_NEED > 120 * 1024 ? SMEM_NEED : 120 * 1024;
};

template <int DH>
__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a, float scale_log2) {
  using namespace attn;
  using Lay = AttnLayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb0 = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  const uint32_t bar0 = smem_u32(bars);
  // barrier slots
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (3 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (5 + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (7 + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (9 + b); };
  auto s_empty = [&](int b) { return bar0 + 8u * (11 + b); };
  const uint32_t p_full = bar0 + 8u * 13;
  const uint32_t pv_done = bar0 + 8u * 14;
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
      mbar_init(s_full(s), 1); mbar_init(s_empty(s), 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
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
  const uint32_t O_COL = 256;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      bool ok = true;
      uint32_t filled = 0;  // bit s: K stage s, bit 2+s: V stage s, bit 4: Q; bit 5+: last parity
      uint32_t fill_ph = 0;
      mbar_arrive_expect_tx(q_full, Lay::TILE);
      for (int b = 0; b < Lay::NBOX; ++b)
        tma_load_3d(sb0 + Lay::Q_OFF + b * BOX, &tm, q_full, b * 64, qt * BQ, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (*abort_flag || !mbar_wait(k_empty(s), ph ^ 1u, a.err, ERR_WAIT_MMA)) { ok = false; break; }
        mbar_arrive_expect_tx(k_full(s), Lay::TILE);
        for (int b = 0; b < Lay::NBOX; ++b)
          tma_load_3d(sb0 + Lay::K_OFF + s * Lay::TILE + b * BOX, &tm, k_full(s), b * 64, j * BKV, BH + bh);
        filled |= 1u << s;
        fill_ph = (fill_ph & ~(1u << s)) | (ph << s);
        if (*abort_flag || !mbar_wait(v_empty(s), ph ^ 1u, a.err, ERR_WAIT_MMA)) { ok = false; break; }
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
        for (int s = 0; s < 2; ++s) {  // tail: all issued tiles consumed
          if (filled & (1u << s)) mbar_wait(k_empty(s), (fill_ph >> s) & 1u, a.err, ERR_WAIT_MMA);
          if (filled & (4u << s)) mbar_wait(v_empty(s), (fill_ph >> (2 + s)) & 1u, a.err, ERR_WAIT_MMA);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      bool ok = mbar_wait(q_full, 0, a.err, ERR_WAIT_TMA);
      bool any = false;
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        if (*abort_flag || !mbar_wait(p_full, i & 1, a.err, ERR_WAIT_EPI)) return false;
        if (!mbar_wait(v_full(s), (i >> 1) & 1, a.err, ERR_WAIT_TMA)) return false;
        tc_fence_after();
        const uint32_t p_addr = sb0 + Lay::P_OFF;
        const uint32_t v_addr = sb0 + Lay::V_OFF + s * Lay::TILE;
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(p_addr + (k >> 2) * BOX + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(v_addr + k * 2048, BOX, 1024);
          mma_f16(tmem + O_COL, ad, bd, IDESC_PV, (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(v_empty(s));
        tc_commit(pv_done);
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const int sb = j & 1;
        if (*abort_flag || !mbar_wait(k_full(s), (j >> 1) & 1, a.err, ERR_WAIT_TMA)) { ok = false; break; }
        if (!mbar_wait(s_empty(sb), ((j >> 1) & 1) ^ 1u, a.err, ERR_WAIT_EPI)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = sb0 + Lay::Q_OFF;
        const uint32_t k_addr = sb0 + Lay::K_OFF + s * Lay::TILE;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(q_addr + (k >> 2) * BOX + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + (k >> 2) * BOX + (k & 3) * 32, 16, 1024);
          mma_f16(tmem + sb * BKV, ad, bd, IDESC_S, k > 0 ? 1u : 0u);
        }
        any = true;
        tc_commit(k_empty(s));
        tc_commit(s_full(sb));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(nkv - 1);
      if (!ok) {
        *abort_flag = 1;
        if (any) {
          tc_commit(drain);
          mbar_wait(drain, 0, a.err, ERR_WAIT_DRAIN, kDrainLimitNs);
        }
      }
    }
  } else {
    // ---------------- softmax warps 2..5: thread = query row
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_lane = (uint32_t)(quad * 32) << 16;
    uint8_t* P = smem + Lay::P_OFF;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      // tcgen05.ld/st are warp-collective (.sync.aligned): every decision that
      // guards them is made uniform across the warp.
      const bool s_ok = !*abort_flag && mbar_wait(s_full(sb), (j >> 1) & 1, a.err, ERR_WAIT_MMA);
      if (!__all_sync(0xFFFFFFFFu, s_ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c)
        tmem_ld32(tmem + t_lane + sb * BKV + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty(sb));

      const int nvalid = min(BKV, L - j * BKV);
      float mx = -INFINITY;
      if (nvalid == BKV) {
#pragma unroll
        for (int i = 0; i < BKV; ++i) mx = fmaxf(mx, __uint_as_float(sr[i]));
      } else {
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (i < nvalid) mx = fmaxf(mx, __uint_as_float(sr[i]));
      }
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
      float rowsum = 0.0f;
#pragma unroll
      for (int i = 0; i < BKV; i += 2) {
        float p0 = fast_exp2(fmaf(__uint_as_float(sr[i]), scale_log2, -m_run));
        float p1 = fast_exp2(fmaf(__uint_as_float(sr[i + 1]), scale_log2, -m_run));
        if (nvalid < BKV) {
          if (i >= nvalid) p0 = 0.0f;
          if (i + 1 >= nvalid) p1 = 0.0f;
        }
        const uint32_t pk = pack_bf16x2(p0, p1);
        rowsum += bf16_lo(pk) + bf16_hi(pk);
        sr[i >> 1] = pk;  // packed P overwrites the consumed scores
      }
      l_run = fmaf(l_run, alpha, rowsum);

      const bool pv_ok = (j == 0) || mbar_wait(pv_done, (j - 1) & 1, a.err, ERR_WAIT_MMA);
      if (!__all_sync(0xFFFFFFFFu, pv_ok)) { ok = false; break; }
      // The whole warp rescales its rows of O if any row's max moved; rows that
      // kept their max use alpha = 1.
      if (__any_sync(0xFFFFFFFFu, rescale)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + t_lane + O_COL + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem + t_lane + O_COL + c * 32, o);
        }
        tmem_st_wait();
      }
      // P row -> shared memory, K-major 128-byte-swizzled operand layout:
      // keys [64b, 64b+64) of row r live in box b at r*128, 16-byte chunk c at (c ^ (r & 7)).
#pragma unroll
      for (int ch = 0; ch < BKV / 8; ++ch) {
        const int b = ch >> 3, c = ch & 7;
        uint4* dst = reinterpret_cast<uint4*>(P + b * BOX + row * 128 + ((c ^ (row & 7)) << 4));
        *dst = make_uint4(sr[4 * ch], sr[4 * ch + 1], sr[4 * ch + 2], sr[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    const bool fin = ok && mbar_wait(pv_done, (nkv - 1) & 1, a.err, ERR_WAIT_MMA);
    if (__all_sync(0xFFFFFFFFu, fin)) {
      tc_fence_after();
      const int q = qt * BQ + row;
      const int b = bh / a.n_heads, h = bh - b * a.n_heads;
      const float inv_l = 1.0f / l_run;
      float amax = 0.0f;
      const int dm = a.n_heads * DH;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.o) + ((size_t)b * L + q) * dm + h * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + t_lane + O_COL + c * 32, o);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
          amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(pk[e])), fabsf(bf16_hi(pk[e]))));
        }
        if (q < L) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int g = 0; g < 4; ++g) d4[g] = make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
        }
      }
      if (q < L) atomicMax(reinterpret_cast<unsigned*>(a.absmax) + (size_t)b * L + q, __float_as_uint(amax));
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

template <int DH>
static cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  using Lay = AttnLayout<DH>;
  CUtensorMap tm;
  // qkv viewed as [3*B*H][L][DH]
  if (!make_tmap_3d(&tm, a.qkv, 2, (uint64_t)DH, (uint64_t)a.L, (uint64_t)3 * a.B * a.n_heads, 64, attn::BKV))
    return cudaErrorInvalidValue;
  auto k = attention_kernel<DH>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.L + attn::BQ - 1) / attn::BQ, a.B * a.n_heads);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  k<<<grid, attn::kThreads, Lay::SMEM, st>>>(tm, a, scale_log2);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.L == 0 || a.B == 0) return cudaSuccess;
  if (a.head_dim == 128) return launch_attn<128>(a, st);
  if (a.head_dim == 64) return launch_attn<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace h3b
