// Tensor-core GEMM for the block's projections on sm_100a:
//   C[m][n] = sum_k A[m][k] * W[n][k]
// with int8 operands (tcgen05.mma kind::i8, exact int32 accumulation) or bf16
// operands (kind::f16, fp32 accumulation), and the block's epilogues fused:
// per-token x per-channel dequantization, QKV with 3D RoPE written head-major,
// GELU with the per-row absmax the next quantizer needs, and the gated
// residual update of the bf16 residual stream.
//
// Method references (web pages on the h3.c / h3-metal engine):
//   "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론", section "Int8 양자화"
//     (int8 MLP and QKV; per-output-channel weight scales, per-row dynamic
//     activation scales) and section "Metal 4 및 TensorOps" (Q/K/V routed
//     directly into a head-major attention input).
//   "h3.c與MLX路線對比：MiniMax-H3在Apple Silicon上的兩種推理實現工程取捨",
//     section "性能上限" (RoPE folded into the kernel of the projections).
//
// Design (B200): persistent kernel on CTA pairs (clusters of two), one 256x256
// output tile at a time per pair, tiles rastered in L2-sized groups (a band of
// A stripes or of W slices stays resident). In each CTA warp 0 streams its 128
// rows of A and its 128 of the tile's 256 W rows with TMA (128-byte swizzle)
// into a 6-stage shared-memory ring, so that an SM pulls 32 KB per K step
// instead of the 48 KB of a one-CTA 128x256 tile (the L2-to-shared-memory feed
// bounded that one near 78% of the MMA rate); warp 1 of the even CTA issues
// tcgen05.mma (cta_group::2, M = 256) from one thread into each CTA's
// double-buffered TMEM accumulator (2 x 256 columns); warps 2-9 (two per
// sub-partition, each half of the columns) drain the other accumulator
// (tcgen05.ld) and run the epilogue while the next tile's MMAs proceed: each
// warp stages its columns' weight scales, bias and gate in shared memory before
// the accumulator wait, requests the next 32 accumulator columns before
// processing the current ones, and (QKV) reads the RoPE table from shared
// memory. The bf16 row-major outputs (dequant, GELU, gated residual) leave
// through TMA tile stores from a per-warp 32 x 32 staging box, and the gated
// residual's x arrives by coalesced loads that the same box turns into rows.
// Every wait is bounded.
#include <atomic>

#include "h3b_common.cuh"
#include "h3b_internal.h"

namespace h3b {
namespace gemm {
constexpr int BM = 128, BN = 256, BKB = 128, STAGES = 4;
constexpr int A_BYTES = BM * BKB;
constexpr int B_BYTES = BN * BKB;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// CTA pairs: per CTA and stage its 128 rows of A and its 128 of the tile's 256 B
// rows, six stages in the same shared memory as the single-CTA ring
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_STAGE_BYTES = 2 * BM * BKB;
static_assert(PAIR_STAGES * PAIR_STAGE_BYTES == STAGES * STAGE_BYTES, "same shared-memory layout");
constexpr int kEpiWarps = 8;  // two per sub-partition, each half of the tile's columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr size_t kL2Budget = 32ull << 20;  // operand bytes the raster keeps resident in L2
constexpr uint32_t TMEM_COLS = 512;
constexpr int kBars = 2 * PAIR_STAGES + 4 + 1;  // enough for either ring
constexpr size_t CONST_OFF = (size_t)STAGES * STAGE_BYTES + 256;     // per-warp epilogue constants
constexpr size_t ROPE_OFF = CONST_OFF + kEpiWarps * 3 * 128 * 4;     // RoPE table, when it fits
constexpr size_t SMEM_BASE = ROPE_OFF + 1024;                         // + 1024 for the alignment slack
// bf16 row-major epilogues: per epilogue warp one 32-row x 32-column staging box
// (64-byte swizzle) that a TMA store writes out; in place of the RoPE table
constexpr int STG_BYTES = 32 * 32 * 2;
constexpr size_t STG_OFF = (ROPE_OFF + 1023) & ~size_t(1023);
constexpr size_t SMEM_STG = STG_OFF + kEpiWarps * STG_BYTES + 1024;
constexpr size_t kSmemMax = 227 * 1024;
static_assert(SMEM_STG <= kSmemMax, "staging boxes fit");
constexpr int kRopeSmemMaxEntries = (int)((kSmemMax - SMEM_BASE) / 8);
}  // namespace gemm

// Tile t -> (M-tile, N-tile). Tiles are rastered in groups: `group` M-tiles
// with the M index fastest (their A stripes stay in L2 while W streams), or
// `group` N-tiles with the N index fastest (their W slices stay resident
// while A streams).
__device__ __forceinline__ void tile_coords(int t, int n_m, int n_n, int raster_n, int group, int& mb,
                                            int& nb) {
  if (!raster_n) {
    const int per_group = group * n_n;
    const int g = t / per_group;
    const int first = g * group;
    const int gm = min(group, n_m - first);
    const int r = t - g * per_group;
    mb = first + r % gm;
    nb = r / gm;
  } else {
    const int per_group = group * n_m;
    const int g = t / per_group;
    const int first = g * group;
    const int gn = min(group, n_n - first);
    const int r = t - g * per_group;
    nb = first + r % gn;
    mb = r / gn;
  }
}

// GELU, tanh form: 0.5 x (1 + tanh(u)) = x / (1 + exp(-2u)) with
// u = sqrt(2/pi) (x + 0.044715 x^3), i.e. x / (1 + 2^(x (k1 + k2 x^2))) with
// k1 = -2 sqrt(2/pi) log2(e), k2 = 0.044715 k1. For very negative x the power
// overflows and the fast reciprocal returns the limit 0.
constexpr float kGeluK1 = -2.0f * 0.7978845608028654f * 1.4426950408889634f;
constexpr float kGeluK2 = 0.044715f * kGeluK1;
__device__ __forceinline__ float2 gelu_tanh2(float2 x) {
  const float2 x2 = __fmul2_rn(x, x);
  const float2 t = __fmul2_rn(x, __ffma2_rn(x2, make_float2(kGeluK2, kGeluK2), make_float2(kGeluK1, kGeluK1)));
  float e0, e1;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(t.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(t.y));
  return make_float2(__fdividef(x.x, 1.0f + e0), __fdividef(x.y, 1.0f + e1));
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32], int valid) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    if (g * 8 >= valid) break;
    d4[g] = make_uint4(pack_bf16x2(v[8 * g + 0], v[8 * g + 1]), pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                       pack_bf16x2(v[8 * g + 4], v[8 * g + 5]), pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
  }
}

// The residual x of a warp's 32 rows x 128 columns, loaded before the accumulator
// is ready so the global-memory latency overlaps the K loop. The loads are
// coalesced: for chunk i (32 columns) and row group j, lane l reads row
// r0 + 8 j + l / 4, columns 32 i + 8 (l % 4) .. + 7 (eight rows of 64 bytes per
// instruction); the epilogue turns them into one row per thread through the
// warp's staging box.
constexpr int kResidVecs = 16;  // 4 chunks x 4 row groups of 16 bytes
__device__ __forceinline__ void prefetch_resid(const GemmArgs& p, int r0, int n0, int lane, uint4 (&xp)[kResidVecs]) {
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.out);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = r0 + 8 * j + (lane >> 2);
      const int col = n0 + 32 * i + 8 * (lane & 3);
      xp[4 * i + j] = (row < p.M && col < p.N &&
                       H3B_IDX_OK((long long)row * p.N + col + 7, (long long)p.M * p.N, p.err))
                          ? *reinterpret_cast<const uint4*>(x + (size_t)row * p.N + col)
                          : make_uint4(0, 0, 0, 0);
    }
}

// Per-warp column constants of the current tile (the warp's 128 columns):
// weight scale, bias and (gated residual) gate, staged in shared memory before
// the accumulator wait so the epilogue reads them at shared-memory latency.
struct EpiConst {
  float sw[128];
  float bias[128];
  float gate[128];
};

template <bool kInt8, int kEpi>
__device__ __forceinline__ void stage_constants(const GemmArgs& p, EpiConst& ec, int col0, int first_row, int lane) {
  // four consecutive columns per lane; N is a multiple of 8, so a float4 is in or out as a whole
  const int c = col0 + 4 * lane;
  const bool ok = c < p.N;
  if (kInt8 && kEpi != EPI_S32)
    *reinterpret_cast<float4*>(&ec.sw[4 * lane]) = ok ? __ldg(reinterpret_cast<const float4*>(p.sW + c))
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
  if (kEpi != EPI_S32 && p.bias)
    *reinterpret_cast<float4*>(&ec.bias[4 * lane]) = ok ? __ldg(reinterpret_cast<const float4*>(p.bias + c))
                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
  if (kEpi == EPI_RESID) {
    const int item = min(first_row, p.M - 1) / p.rows_per_item;
    *reinterpret_cast<float4*>(&ec.gate[4 * lane]) =
        ok ? __ldg(reinterpret_cast<const float4*>(p.gate + (size_t)item * p.gate_stride + c))
           : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// The bf16 row-major outputs (dequant, GELU, gated residual) leave through TMA
// stores: a warp's 32 rows x 32 columns go to its staging box, thread = row, the
// 16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3) (the 64-byte swizzle,
// which also spreads a quarter-warp's eight 16-byte writes over all banks), and
// one lane stores the box. The hardware clips rows >= M and columns >= N.
template <int kEpi>
constexpr bool tma_store_epi() { return kEpi == EPI_DEQ || kEpi == EPI_GELU || kEpi == EPI_RESID; }

// Byte offset of the 16-byte chunk c of row r in a staging box.
__device__ __forceinline__ uint32_t stg_off(uint32_t r, uint32_t c) { return r * 64u + 16u * (c ^ ((r >> 1) & 3u)); }

// The previous box of this warp has been read out of the staging buffer.
__device__ __forceinline__ void stage_acquire(int lane) {
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
}

// Chunk i of the coalesced residual prefetch into the staging box, then this
// thread's row of it (the box must have been acquired).
__device__ __forceinline__ void stage_resid_row(uint32_t stg, const uint4 (&xp)[kResidVecs], int i, int lane,
                                                uint4 (&xr)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 v = xp[4 * i + j];
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg + stg_off(8u * j + ((uint32_t)lane >> 2), lane & 3u)),
                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
  }
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 4; ++c)
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(xr[c].x), "=r"(xr[c].y), "=r"(xr[c].z), "=r"(xr[c].w)
                 : "r"(stg + stg_off((uint32_t)lane, (uint32_t)c))
                 : "memory");
}

// This thread's row of the chunk into the staging box and one lane's TMA store
// of the box (the box must have been acquired; a thread overwrites only the
// positions of its own row).
__device__ __forceinline__ void stage_and_store(const CUtensorMap* tmC, uint32_t stg, const uint32_t (&pk)[16],
                                                int lane, int col0, int r0, bool rows_in) {
  const uint32_t rowaddr = stg + (uint32_t)lane * 64u;
  const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowaddr + 16u * ((uint32_t)c ^ sw)),
                 "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                 : "memory");
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && rows_in) {
    tma_store_2d(tmC, stg, col0, r0);
    bulk_commit_group();
  }
}

// Epilogue of the warp's 32 rows x 128 columns of one 128x256 tile; the thread
// owns TMEM lane = tile row. TMEM loads are double-buffered: chunk i+1 (32
// columns) is requested before chunk i is processed. `rope_s` is the RoPE
// table in shared memory (or the global table when it did not fit). `r0` is
// the warp's first row; `stg` its staging box for the TMA-stored outputs.
template <bool kInt8, int kEpi>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& p, uint32_t tbase, int row, bool row_ok, int n0,
                                              const EpiConst& ec, bool gate_uniform, const float2* rope_s,
                                              const uint4 (&xp)[kResidVecs], const CUtensorMap* tmC,
                                              uint32_t stg, int r0) {
  constexpr bool kTmaStore = tma_store_epi<kEpi>();
  float sa = 1.0f;
  if (kInt8 && kEpi != EPI_S32 && row_ok) sa = __ldg(p.sA + row);
  int item = 0, l = 0, pt = 0, ph = 0, pw = 0;
  if (kEpi == EPI_QKV) {
    item = row / p.L;
    l = row - item * p.L;
    pt = l / (p.H * p.W);
    ph = (l / p.W) % p.H;
    pw = l % p.W;
  } else if (kEpi == EPI_RESID) {
    item = row / p.rows_per_item;
  }
  float amax = 0.0f;
  // the gated residual holds its prefetched x (16 vectors per thread) in the
  // registers a second accumulator chunk would take, so it loads one chunk at a time
  constexpr bool kDoubleBuffer = kEpi != EPI_RESID;
  uint32_t r[kDoubleBuffer ? 2 : 1][32];
  tmem_ld32(tbase, r[0]);
  tmem_ld_wait();
  tmem_reg_fence(r[0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int col0 = n0 + i * 32;
    if (col0 >= p.N) break;  // uniform across the warp
    const bool next = i + 1 < 4 && col0 + 32 < p.N;
    if (kDoubleBuffer && next) tmem_ld32(tbase + (i + 1) * 32, r[(i + 1) & 1]);
    const uint32_t (&rc)[32] = r[kDoubleBuffer ? (i & 1) : 0];
    uint32_t pk[16];  // the chunk as bf16 pairs, for the TMA store (zero in rows past M)
    uint4 xr[4];      // gated residual: this row's 32 columns of x
    if (kTmaStore) {
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = 0u;
      if (kEpi == EPI_RESID) {
        stage_acquire(threadIdx.x & 31);
        stage_resid_row(stg, xp, i, threadIdx.x & 31, xr);
      }
    }
    if (row_ok) {
      const int valid = min(32, p.N - col0);
      if (kEpi == EPI_S32) {
        uint4* d4 = reinterpret_cast<uint4*>(static_cast<int32_t*>(p.out) + (size_t)row * p.N + col0);
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (g * 4 < valid && H3B_IDX_OK((long long)row * p.N + col0 + 4 * g + 3, (long long)p.M * p.N, p.err))
            d4[g] = make_uint4(rc[4 * g], rc[4 * g + 1], rc[4 * g + 2], rc[4 * g + 3]);
      } else {
        float v[32];
        if (kInt8) {
          const float2 sa2 = make_float2(sa, sa);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 sw = *reinterpret_cast<const float4*>(&ec.sw[i * 32 + 4 * g]);
            const float2 lo = __fmul2_rn(__fmul2_rn(make_float2((float)(int)rc[4 * g], (float)(int)rc[4 * g + 1]), sa2),
                                         make_float2(sw.x, sw.y));
            const float2 hi = __fmul2_rn(__fmul2_rn(make_float2((float)(int)rc[4 * g + 2], (float)(int)rc[4 * g + 3]), sa2),
                                         make_float2(sw.z, sw.w));
            v[4 * g + 0] = lo.x; v[4 * g + 1] = lo.y; v[4 * g + 2] = hi.x; v[4 * g + 3] = hi.y;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(rc[e]);
        }
        if (p.bias) {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 b = *reinterpret_cast<const float4*>(&ec.bias[i * 32 + 4 * g]);
            v[4 * g] += b.x; v[4 * g + 1] += b.y; v[4 * g + 2] += b.z; v[4 * g + 3] += b.w;
          }
        }
        if (kEpi == EPI_DEQ) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        } else if (kEpi == EPI_GELU) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 gv = gelu_tanh2(make_float2(v[e], v[e + 1]));
            v[e] = round_bf16(gv.x);
            v[e + 1] = round_bf16(gv.y);
            amax = fmaxf(amax, fmaxf(fabsf(v[e]), fabsf(v[e + 1])));
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        } else if (kEpi == EPI_RESID) {
          const float* gsrc = gate_uniform ? &ec.gate[i * 32] : p.gate + (size_t)item * p.gate_stride + col0;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (g * 8 >= valid) break;
            const uint4 xv = xr[g];
            float4 ga, gb;
            if (gate_uniform) {
              ga = *reinterpret_cast<const float4*>(gsrc + 8 * g);
              gb = *reinterpret_cast<const float4*>(gsrc + 8 * g + 4);
            } else {
              ga = __ldg(reinterpret_cast<const float4*>(gsrc + 8 * g));
              gb = __ldg(reinterpret_cast<const float4*>(gsrc + 8 * g + 4));
            }
            const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              v[8 * g + 2 * e] = fmaf(gg[2 * e], v[8 * g + 2 * e], bf16_lo(xu[e]));
              v[8 * g + 2 * e + 1] = fmaf(gg[2 * e + 1], v[8 * g + 2 * e + 1], bf16_hi(xu[e]));
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        } else if (kEpi == EPI_QKV) {
          const int part = col0 / p.d;
          const int rem = col0 - part * p.d;
          const int head = rem / p.head_dim;
          const int lane0 = rem - head * p.head_dim;
          if (part < 2) {
            const int off_h = p.T * (p.rope_t / 2), off_w = off_h + p.H * (p.rope_h / 2);
            const int base_t = pt * (p.rope_t / 2), base_h = off_h + ph * (p.rope_h / 2) - p.rope_t / 2,
                      base_w = off_w + pw * (p.rope_w / 2) - (p.rope_t + p.rope_h) / 2;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int pl = lane0 + 2 * e;
              const int idx = (pl < p.rope_t ? base_t : (pl < p.rope_t + p.rope_h ? base_h : base_w)) + (pl >> 1);
              const float2 cs = rope_s[idx];
              const float x0 = v[2 * e], x1 = v[2 * e + 1];
              v[2 * e] = x0 * cs.x - x1 * cs.y;
              v[2 * e + 1] = x0 * cs.y + x1 * cs.x;
            }
          }
          const size_t off = ((((size_t)part * p.B + item) * p.n_heads + head) * p.L + l) * p.head_dim + lane0;
          if (H3B_IDX_OK((long long)off + 31, (long long)p.M * p.N, p.err))
            store_bf16x32(static_cast<__nv_bfloat16*>(p.out) + off, v, 32);
        }
      }
    }
    if (kTmaStore) {
      if (kEpi != EPI_RESID) stage_acquire(threadIdx.x & 31);
      stage_and_store(tmC, stg, pk, threadIdx.x & 31, col0, r0, r0 < p.M);
    }
    if (next) {
      if (!kDoubleBuffer) tmem_ld32(tbase + (i + 1) * 32, r[0]);
      tmem_ld_wait();
      tmem_reg_fence(r[kDoubleBuffer ? ((i + 1) & 1) : 0]);
    }
  }
  if (kEpi == EPI_GELU && row_ok)
    atomicMax(reinterpret_cast<unsigned*>(p.absmax) + row, __float_as_uint(amax));
}

// kPair: the CTA is one of a pair (cluster of two) that computes 256 x 256
// tiles: rank r takes rows [256 mb + 128 r, +128) of A and rows [256 nb + 128 r,
// +128) of W into its shared memory, the even CTA issues every MMA for both
// (M = 256, cta_group::2) and commits to both CTAs' barriers, and each CTA's
// epilogue drains its own 128 x 256 accumulator. The stage's bytes of both CTAs
// complete on the even CTA's full barrier; both CTAs' epilogues release an
// accumulator on the even CTA's tempty barrier.
template <bool kInt8, int kEpi, bool kPair>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const GemmArgs p) {
  using namespace gemm;
  constexpr int NS = kPair ? PAIR_STAGES : STAGES;
  constexpr int SB = kPair ? PAIR_STAGE_BYTES : STAGE_BYTES;
  constexpr int MT = kPair ? 2 * BM : BM;  // tile rows
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NS * SB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBars);
  EpiConst* epi_const = reinterpret_cast<EpiConst*>(smem + CONST_OFF);
  float2* rope_smem = reinterpret_cast<float2*>(smem + ROPE_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (NS + s); };
  auto tfull = [&](int a) { return bar0 + 8u * (2 * NS + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (2 * NS + 2 + a); };
  const uint32_t drain = bar0 + 8u * (2 * NS + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  // an abort in either CTA of a pair ends the waits of both
  auto set_abort = [&]() {
    *abort_flag = 1;
    if (kPair) {
      const uint32_t peer = mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u);
      asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
    }
  };
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // pair or CTA
  const int units = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int n_m = (p.M + MT - 1) / MT, n_n = (p.N + BN - 1) / BN;
  const int n_tiles = n_m * n_n;
  constexpr int BKE = kInt8 ? BKB : BKB / 2;  // K elements per stage
  const int nk = (p.K + BKE - 1) / BKE;
  constexpr uint32_t IDESC = kInt8 ? instr_desc(2, 1, 0, 0, MT, BN) : instr_desc(1, 1, 0, 0, MT, BN);
  constexpr uint32_t B_ROWS = kPair ? BN / 2 : BN;  // W rows of a stage in this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull(a), 1); mbar_init(tempty(a), (kPair ? 2 : 1) * kEpiWarps); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (tma_store_epi<kEpi>()) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
    tc_fence_before();
  }
  __syncthreads();
  if (kPair) cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // A (and the residual x) come from earlier grids
  griddep_launch_dependents();
  if (kEpi == EPI_QKV && p.rope_smem_entries > 0) {  // the whole RoPE table, once per CTA
    for (int i = threadIdx.x; i < p.rope_smem_entries; i += blockDim.x) rope_smem[i] = __ldg(p.rope + i);
    __syncthreads();
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (in both CTAs of a pair)
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_ph = 0;  // per-stage bitmask of the last issued phase
      bool ok = true;
      for (int t = unit; t < n_tiles && ok; t += units) {
        int mb, nb;
        tile_coords(t, n_m, n_n, p.raster_n, p.group, mb, nb);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_or_abort(empty(s), ph ^ 1u, abort_flag, p.err, ERR_WAIT_MMA)) { ok = false; break; }
          const uint32_t a_dst = sbase + s * SB;
          if (kPair) {
            if (leader) mbar_arrive_expect_tx(full(s), 2 * SB);
            const uint32_t fb = mapa_shared(full(s), 0);
            tma_load_2d_pair(a_dst, &tmA, fb, kb * BKE, mb * MT + (int)rank * BM);
            tma_load_2d_pair(a_dst + A_BYTES, &tmB, fb, kb * BKE, nb * BN + (int)rank * (int)B_ROWS);
          } else {
            mbar_arrive_expect_tx(full(s), SB);
            tma_load_2d(a_dst, &tmA, full(s), kb * BKE, mb * MT);
            tma_load_2d(a_dst + A_BYTES, &tmB, full(s), kb * BKE, nb * BN);
          }
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
          if (++s == NS) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        set_abort();
        if (leader)  // let in-flight tiles land before the CTA exits (a pair's full barriers count both CTAs)
          for (int i = 0; i < NS; ++i)
            if (issued & (1u << i)) mbar_wait(full(i), (issued_ph >> i) & 1u, p.err, ERR_WAIT_DRAIN, kDrainLimitNs);
      } else {
        // tail: every filled stage has been consumed (its commit has arrived)
        for (int i = 0; i < NS; ++i)
          if (issued & (1u << i)) mbar_wait(empty(i), (issued_ph >> i) & 1u, p.err, ERR_WAIT_MMA);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the even CTA of a pair issues for both)
      int s = 0;
      uint32_t ph = 0;
      int tl = 0;
      bool ok = true;
      bool any = false;
      for (int t = unit; t < n_tiles && ok; t += units, ++tl) {
        const int acc = tl & 1;
        const uint32_t aph = (tl >> 1) & 1;
        if (!mbar_wait_or_abort(tempty(acc), aph ^ 1u, abort_flag, p.err, ERR_WAIT_EPI)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_or_abort(full(s), ph, abort_flag, p.err, ERR_WAIT_TMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = sbase + s * SB;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = smem_desc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(a_addr + A_BYTES + k * 32, 16, 1024);
            const uint32_t accum = (kb | k) != 0;
            if (kPair) {
              if (kInt8) mma_i8_pair(d_tmem, ad, bd, IDESC, accum);
              else mma_f16_pair(d_tmem, ad, bd, IDESC, accum);
            } else {
              if (kInt8) mma_i8(d_tmem, ad, bd, IDESC, accum);
              else mma_f16(d_tmem, ad, bd, IDESC, accum);
            }
          }
          any = true;
          if (kPair) tc_commit_pair(empty(s));
          else tc_commit(empty(s));
          if (++s == NS) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (kPair) tc_commit_pair(tfull(acc));
        else tc_commit(tfull(acc));
      }
      if (!ok) {
        set_abort();
        if (any) {  // wait for the MMAs already issued before TMEM is released
          if (kPair) tc_commit_pair_local(drain);
          else tc_commit(drain);
          mbar_wait(drain, 0, p.err, ERR_WAIT_DRAIN, kDrainLimitNs);
        }
      }
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quadrant = warp % 4; warps
    // 2-5 take columns [0, 128) of the tile, warps 6-9 columns [128, 256)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tempty_leader0 = kPair ? mapa_shared(tempty(0), 0) : tempty(0);
    const uint32_t tempty_leader1 = kPair ? mapa_shared(tempty(1), 0) : tempty(1);
    int tl = 0;
    for (int t = unit; t < n_tiles; t += units, ++tl) {
      int mb, nb;
      tile_coords(t, n_m, n_n, p.raster_n, p.group, mb, nb);
      const int acc = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      const int r0 = mb * MT + (int)rank * BM + quad * 32;  // this warp's first row
      const int row = r0 + lane;
      const int n0 = nb * BN + half * (BN / 2);
      EpiConst& ec = epi_const[warp - 2];
      // this warp finished its previous tile, so its constants buffer is free
      stage_constants<kInt8, kEpi>(p, ec, n0, r0, lane);
      const int first_row = min(r0, p.M - 1), last_row = min(r0 + 31, p.M - 1);
      const bool gate_uniform = kEpi == EPI_RESID && first_row / p.rows_per_item == last_row / p.rows_per_item;
      uint4 xp[kResidVecs];
      if (kEpi == EPI_RESID) prefetch_resid(p, r0, n0, lane, xp);
      __syncwarp();
      // tcgen05.ld is warp-collective: the wait outcome is made warp-uniform.
      const bool t_ok = mbar_wait_or_abort(tfull(acc), aph, abort_flag, p.err, ERR_WAIT_MMA);
      if (!__all_sync(0xFFFFFFFFu, t_ok)) {
        if (lane == 0) set_abort();
        break;
      }
      tc_fence_after();
      // this warp's 32 lanes and 128 columns of the accumulator
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN + half * (BN / 2);
      epilogue_tile<kInt8, kEpi>(p, tbase, row, row < p.M, n0, ec, gate_uniform,
                                 p.rope_smem_entries > 0 ? rope_smem : p.rope, xp, &tmC,
                                 sbase + (uint32_t)STG_OFF + (uint32_t)(warp - 2) * STG_BYTES, r0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kPair) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        else mbar_arrive(tempty(acc));
      }
    }
    // the staging boxes are read and the stores written before the CTA exits
    if (tma_store_epi<kEpi>() && lane == 0) bulk_wait_group0();
  }
  __syncthreads();
  if (kPair) cluster_sync_all();  // the pair's MMAs and remote arrivals are over before TMEM goes
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <bool kInt8, int kEpi, bool kPair>
static cudaError_t launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                              const GemmArgs& a, int grid, cudaStream_t st) {
  auto k = gemm_kernel<kInt8, kEpi, kPair>;
  const size_t smem = tma_store_epi<kEpi>() ? gemm::SMEM_STG
                                            : gemm::SMEM_BASE + (size_t)a.rope_smem_entries * sizeof(float2);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm::kSmemMax);
  if (e != cudaSuccess) return e;
  if (!kPair) return launch_pdl(k, dim3(grid), dim3(gemm::kThreads), smem, st, ta, tb, tc, a);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(gemm::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below sees the cluster shape only
  // persistent pairs: no more than can be resident at once (looked up once per device;
  // the shared-memory size the launcher asks for does not change the answer)
  constexpr int kMaxDevices = 64;
  static std::atomic<int> resident[kMaxDevices];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int clusters = dev >= 0 && dev < kMaxDevices ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (clusters < 1) {
    cfg.dynamicSmemBytes = gemm::kSmemMax;  // the most the kernel asks for
    e = cudaOccupancyMaxActiveClusters(&clusters, k, &cfg);
    cfg.dynamicSmemBytes = smem;
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < kMaxDevices) resident[dev].store(clusters, std::memory_order_relaxed);
  }
  if ((int)cfg.gridDim.x > 2 * clusters) cfg.gridDim.x = 2u * (unsigned)clusters;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k, ta, tb, tc, a);
}

// The GEMMs run on CTA pairs (256 x 256 tiles, half of every W tile per SM) when
// the GPU has at least two SMs and the problem at least one pair tile.
constexpr bool kUsePairs = true;

template <bool kInt8, int kEpi>
static cudaError_t launch_epi(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                              const GemmArgs& a, bool pair, int grid, cudaStream_t st) {
  return pair ? launch_one<kInt8, kEpi, true>(ta, tb, tc, a, grid, st)
              : launch_one<kInt8, kEpi, false>(ta, tb, tc, a, grid, st);
}

cudaError_t launch_gemm(bool int8_operands, GemmEpilogue epi, const void* A, const void* W,
                        const GemmArgs& a, int sms, cudaStream_t st) {
  using namespace gemm;
  if (a.M == 0) return cudaSuccess;
  const bool pair = kUsePairs && sms >= 2;
  const int MT = pair ? 2 * BM : BM;
  const int eb = int8_operands ? 1 : 2;
  const uint32_t bke = int8_operands ? BKB : BKB / 2;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, eb, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * eb, bke, BM))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, W, eb, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.K * eb, bke, pair ? BN / 2 : BN))
    return cudaErrorInvalidValue;
  // the bf16 [M][N] output of the TMA-stored epilogues: 32 x 32 boxes, 64-byte swizzle
  CUtensorMap tc = tb;
  if ((epi == EPI_DEQ || epi == EPI_GELU || epi == EPI_RESID) &&
      !make_tmap_2d(&tc, a.out, 2, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.N * 2, 32, 32, 64))
    return cudaErrorInvalidValue;
  const int n_m = (a.M + MT - 1) / MT, n_n = (a.N + BN - 1) / BN;
  const int n_tiles = n_m * n_n;
  const int units = pair ? sms / 2 : sms;  // persistent pairs or CTAs
  const int grid = (n_tiles < units ? n_tiles : units) * (pair ? 2 : 1);
  // Raster: keep either a band of A stripes or a band of W slices resident in L2,
  // whichever makes the other operand's repeated streaming cheaper.
  GemmArgs args = a;
  args.rope_smem_entries = 0;
  if (epi == EPI_QKV && a.rope) {
    const int entries = a.T * (a.rope_t / 2) + a.H * (a.rope_h / 2) + a.W * (a.rope_w / 2);
    if (entries <= kRopeSmemMaxEntries) args.rope_smem_entries = entries;
  }
  {
    const double stripe_a = (double)MT * a.K * eb, slice_w = (double)BN * a.K * eb;
    const double bytes_a = (double)a.M * a.K * eb, bytes_w = (double)a.N * a.K * eb;
    int gm = (int)(kL2Budget / stripe_a), gn = (int)(kL2Budget / slice_w);
    gm = gm < 1 ? 1 : (gm > n_m ? n_m : gm);
    gn = gn < 1 ? 1 : (gn > n_n ? n_n : gn);
    const double traffic_m = bytes_a + ((n_m + gm - 1) / gm) * bytes_w;
    const double traffic_n = bytes_w + ((n_n + gn - 1) / gn) * bytes_a;
    args.raster_n = traffic_n < traffic_m ? 1 : 0;
    args.group = args.raster_n ? gn : gm;
  }
  if (int8_operands) {
    switch (epi) {
      case EPI_S32: return launch_epi<true, EPI_S32>(ta, tb, tc, args, pair, grid, st);
      case EPI_DEQ: return launch_epi<true, EPI_DEQ>(ta, tb, tc, args, pair, grid, st);
      case EPI_QKV: return launch_epi<true, EPI_QKV>(ta, tb, tc, args, pair, grid, st);
      case EPI_RESID: return launch_epi<true, EPI_RESID>(ta, tb, tc, args, pair, grid, st);
      case EPI_GELU: return launch_epi<true, EPI_GELU>(ta, tb, tc, args, pair, grid, st);
    }
  } else {
    switch (epi) {
      case EPI_DEQ: return launch_epi<false, EPI_DEQ>(ta, tb, tc, args, pair, grid, st);
      case EPI_QKV: return launch_epi<false, EPI_QKV>(ta, tb, tc, args, pair, grid, st);
      case EPI_RESID: return launch_epi<false, EPI_RESID>(ta, tb, tc, args, pair, grid, st);
      default: break;
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace h3b
