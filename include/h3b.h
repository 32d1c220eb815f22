/*
 * h3b — forward pass of one gated-AdaLN DiT block over video latent tokens, on
 * NVIDIA B200 (sm_100a). C ABI: plain pointers and sizes, no framework types.
 *
 * The method (web pages about the h3.c / h3-metal MiniMax-H3 engine; cited in
 * the entry points below by the short names in brackets):
 *   [README] "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론"
 *       section "Int8 양자화": int8 MLP and QKV with dynamic per-row activation
 *       quantization and per-output-channel weight scales; the activation
 *       quantizer is fused into the preceding gated-AdaLN kernel.
 *       section "Metal 4 및 TensorOps": Q/K/V routed straight into a head-major
 *       attention input.
 *       section "속도 및 품질 트레이드오프" (Token Reduction row): horizontally
 *       adjacent video tokens are paired in the middle blocks.
 *   [MLX] "h3.c與MLX路線對比：MiniMax-H3在Apple Silicon上的兩種推理實現工程取捨"
 *       section "性能上限": AdaLN gating, RoPE and quantization folded into the
 *       kernel ahead of the projections.
 *   [BLOG] "맥북에서 AI 영상 생성 모델 돌리기 - MiniMax H3 로컬 실행과 30초 애니메이션 만들기"
 *       section "int8 이 뭔가요": one F32 scale per output channel (weights),
 *       one F32 scale per row computed at run time (activations).
 * Dimensions, LayerNorm eps, GELU form and the RoPE split are parameters; the
 * pages do not state them.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, owned
 *     by the caller; the library never allocates device memory for the block.
 *     Its only device state is one error word per device (h3b_device_error) and
 *     the fixed 32 MiB scratch array of h3b_block_forward_noalloc, which every
 *     GPU that loads the library holds until the process exits. On the host it
 *     keeps per-device attributes and device addresses, looked up once per
 *     device index: use one CUDA context per device, and do not call
 *     cudaDeviceReset between calls (the cached addresses would be stale).
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream).
 *     Kernels are launched with programmatic stream serialization: a kernel may
 *     start its setup while the kernel before it on the stream finishes, but it
 *     waits for that grid (griddepcontrol.wait) before it reads or writes any
 *     tensor, so stream order is kept for the caller's data. A caller's kernel
 *     launched after a call without that attribute waits as usual; one launched
 *     with it must itself wait before reading the call's outputs. The
 *     environment variable H3B_PDL=0 turns the attribute off.
 *   - bf16 tensors are passed as `void*` (IEEE bfloat16 bit patterns).
 *   - Matrices are row-major. Weights are [out][in] (each output channel's input
 *     weights contiguous).
 *   - Arguments are validated on the host BEFORE any launch; on failure nothing
 *     is launched and a negative h3b_status is returned. Launch failures are
 *     reported as H3B_ERR_CUDA. Kernel faults surface at the caller's next
 *     synchronization, as for any CUDA launch.
 *   - Every device pointer must be 16-byte aligned.
 *   - A step entry point given an empty problem (M, rows or n equal to 0)
 *     returns H3B_OK as soon as its sizes are checked: its pointers are not
 *     inspected (NULL is accepted), the device is not queried and nothing is
 *     launched.
 *   - Device-side waits are bounded. A wait that runs out records a nonzero code
 *     in the device error word and the kernel returns; read it with
 *     h3b_device_error after synchronizing.
 */
#ifndef H3B_H
#define H3B_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define H3B_API __attribute__((visibility("default")))
#else
#define H3B_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* h3b_stream; /* == cudaStream_t */

typedef enum {
  H3B_OK = 0,
  H3B_ERR_ARG = -1,          /* NULL pointer or nonsensical value */
  H3B_ERR_SHAPE = -2,        /* unsupported dimensions */
  H3B_ERR_ALIGN = -3,        /* pointer not 16-byte aligned */
  H3B_ERR_WORKSPACE = -4,    /* workspace smaller than h3b_workspace_size */
  H3B_ERR_ARCH = -5,         /* current device is not compute capability 10.0 */
  H3B_ERR_CUDA = -6,         /* a CUDA runtime/driver call failed */
  H3B_ERR_DEVICE_CHECK = -7  /* the device error word is set */
} h3b_status;

/* Block dimensions.
 *   Latent grid T x H x W per batch item, flattened t-major, then h, then w:
 *   token l = (t*H + h)*W + w, L = T*H*W. B independent batch items.
 *   d = n_heads * head_dim; head_dim in {64, 128}; d % 256 == 0, d <= 8192;
 *   d_ff % 256 == 0, d_ff <= 32768; 1 <= B <= 8; B*L < 2^31 tokens and
 *   B*L*d_ff <= 2^40 (H3B_ERR_SHAPE otherwise, checked without overflow for
 *   any int extents).
 *   RoPE: rope_t + rope_h + rope_w == head_dim, each even (3D RoPE; lanes
 *   [0,rope_t) rotate with t, the next rope_h with h, the rest with w; pair
 *   (2j, 2j+1) of a segment of length r has frequency rope_theta^(-2j/r)).
 *   ln_eps: LayerNorm epsilon (no affine, biased variance).
 *   qkv_int8: 1 = int8 QKV projection (default), 0 = bf16 QKV projection.
 *   wo_bf16:  0 = int8 output projection on the quantized attention output
 *             (default), 1 = bf16 output projection on the bf16 attention output
 *             (the BF16 attention-output projection of the pages' tensor path,
 *             "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론",
 *             section "Metal 4 및 TensorOps"); the quant_o pass is skipped. */
typedef struct {
  int B, T, H, W;
  int d, n_heads, head_dim, d_ff;
  int rope_t, rope_h, rope_w;
  float rope_theta, ln_eps;
  int qkv_int8;
  int wo_bf16;
} h3b_dims;

/* Weights of one block (device pointers). int8 codes with one F32 scale per
 * output channel (quantize them with h3b_quantize_weights). Biases may be NULL
 * (zero). b_ada may be NULL.
 *   w_ada     bf16 [6d][d]   AdaLN Linear; output chunks in order
 *                            shift_attn, scale_attn, gate_attn, shift_mlp,
 *                            scale_mlp, gate_mlp
 *   b_ada     fp32 [6d]
 *   wqkv      int8 [3d][d] + sqkv fp32 [3d]   (qkv_int8 == 1)
 *   wqkv_bf16 bf16 [3d][d]                    (qkv_int8 == 0)
 *   bqkv      fp32 [3d]; output channel o -> part o/d (Q, K, V),
 *             head (o % d)/head_dim, lane o % head_dim
 *   wo int8 [d][d]       + so fp32 [d],    bo fp32 [d]   (wo/so when wo_bf16 == 0)
 *   w1 int8 [d_ff][d]    + s1 fp32 [d_ff], b1 fp32 [d_ff]
 *   w2 int8 [d][d_ff]    + s2 fp32 [d],    b2 fp32 [d]
 *   wo_bf16 bf16 [d][d]                                 (wo_bf16 == 1) */
typedef struct {
  const void* w_ada; const float* b_ada;
  const int8_t* wqkv; const float* sqkv; const void* wqkv_bf16; const float* bqkv;
  const int8_t* wo; const float* so; const float* bo;
  const int8_t* w1; const float* s1; const float* b1;
  const int8_t* w2; const float* s2; const float* b2;
  const void* wo_bf16;
} h3b_block_weights;

H3B_API const char* h3b_status_string(h3b_status s);

/* Human-readable detail of the last failing call on this host thread (the
 * failed check or CUDA call); empty when none. Owned by the library. */
H3B_API const char* h3b_last_error_detail(void);

/* Bytes of scratch workspace h3b_block_forward / h3b_blocks_forward need for
 * these dimensions (regions aliased by lifetime). */
H3B_API h3b_status h3b_workspace_size(const h3b_dims* dims, size_t* bytes);

/* One block forward, in place on the residual stream x (bf16 [B][L][d]).
 * The block of "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론",
 * section "Int8 양자화" (gated AdaLN; int8 QKV and MLP with per-token activation
 * and per-output-channel weight scales; the quantizer fused into the AdaLN
 * kernel), with the head-major Q/K/V of section "Metal 4 및 TensorOps" and the
 * AdaLN/RoPE folding of "h3.c與MLX路線對比：MiniMax-H3在Apple Silicon上的兩種推理
 * 實現工程取捨", section "性能上限":
 *   mod = AdaLN Linear(c)                                  c: fp32 [B][d]
 *   A1,s1 = quant(bf16(LN(x)(1+scale_attn)+shift_attn))    (fused kernel)
 *   Q,K,V = deq(A1 Wqkv^T)+bqkv, 3D RoPE on Q,K, written head-major
 *   O = softmax(Q K^T / sqrt(head_dim)) V   (non-causal, per batch item, head)
 *   x += gate_attn * (deq(quant(O) Wo^T) + bo)
 *   A3,s3 = quant(bf16(LN(x)(1+scale_mlp)+shift_mlp))
 *   G = bf16(GELU_tanh(deq(A3 W1^T)+b1))
 *   x += gate_mlp * (deq(quant(G) W2^T) + b2)
 * ws: device workspace of at least h3b_workspace_size bytes (256-byte aligned). */
H3B_API h3b_status h3b_block_forward(const h3b_dims* dims, const h3b_block_weights* w, const float* c,
                             void* x, void* ws, size_t ws_bytes, h3b_stream stream);

/* Allocation-free block forward (the pages have no counterpart; this exists
 * for callers of this library). Same computation and results as
 * h3b_block_forward, but the scratch lives in a fixed 32 MiB device array
 * inside this library, so the call needs no workspace and allocates nothing
 * (no cudaMalloc/cudaFree or allocating library routine). It is meant for
 * callers that cannot allocate device memory when they run the block: code
 * whose device allocator belongs to a host framework that forbids side
 * allocations, plugin or callback code that only receives input and output
 * pointers, or latency-critical loops where an allocation could block.
 *   - Dimensions whose h3b_workspace_size exceeds 32 MiB are rejected with
 *     H3B_ERR_WORKSPACE before any launch (use h3b_block_forward instead).
 *   - Every GPU that loads this library holds the 32 MiB array until the
 *     process exits.
 *   - The first call on a device checks the device (compute capability 10.0,
 *     else H3B_ERR_ARCH) and looks up the array's device address on it
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is cached per device index (one context per device; no
 *     cudaDeviceReset between calls).
 *   - All calls on a device share the array: calls that overlap on the GPU
 *     (different streams or host threads) race on it; serialize them.
 *   - Nothing in the array needs to start at zero; the block's kernels zero
 *     the region that accumulates on every call. */
H3B_API h3b_status h3b_block_forward_noalloc(const h3b_dims* dims, const h3b_block_weights* w,
                                             const float* c, void* x, h3b_stream stream);

/* n_blocks blocks in sequence on one residual stream x (the denoiser's stack of
 * blocks; each block as in h3b_block_forward); block i uses w[i]
 * (HOST array of n_blocks weight structs holding device pointers) and
 * c + i*B*d (device, fp32 [n_blocks][B][d]). Same workspace as one block. */
H3B_API h3b_status h3b_blocks_forward(const h3b_dims* dims, const h3b_block_weights* w, int n_blocks,
                              const float* c, void* x, void* ws, size_t ws_bytes,
                              h3b_stream stream);

/* Multi-block pass with token reduction over a middle range of blocks (the
 * Token Reduction row of the control table in "h3-metal: ...", section
 * "속도 및 품질 트레이드오프": horizontally adjacent video tokens are paired in
 * the middle blocks).
 * Blocks [0, first) run on the full grid `full`; then the tokens are paired
 * once (h3b_token_pair into ym), blocks [first, last) run on the merged grid
 * (W/2, in place on ym), the block deltas are added back at both positions
 * once (h3b_token_unpair into x, which recomputes the merged input from x),
 * and blocks [last, n_blocks) run on the full grid again.
 *   0 <= first <= last <= n_blocks; full->W even when first < last.
 *   ym: bf16 [B][T][H][W/2][d] device buffer (unused when first == last).
 *   xm: not used (kept for the argument order); may be NULL.
 *   ws: at least h3b_workspace_size(full) bytes (that covers the merged grid).
 *   w, c: as for h3b_blocks_forward. */
H3B_API h3b_status h3b_blocks_forward_reduced(const h3b_dims* full, const h3b_block_weights* w, int n_blocks,
                                              int first, int last, const float* c, void* x, void* xm, void* ym,
                                              void* ws, size_t ws_bytes, h3b_stream stream);

/* Residual reuse across denoise steps (the core-residual reuse of the pages'
 * control table, "h3-metal: ...", section "속도 및 품질 트레이드오프"): the
 * delta a block range [first, last) adds to the residual stream on a fresh
 * denoise step is cached and re-applied on the following steps instead of
 * running the range again.
 *   h3b_blocks_forward_cached: blocks [0, first) and [last, n_blocks) run as in
 *   h3b_blocks_forward. fresh != 0: x is copied to x_save (bf16, B*L*d), the
 *   range runs, then delta = x - x_save (fp32, B*L*d). fresh == 0: the range is
 *   skipped and x = bf16(x + delta). first == last: no range (x_save, delta unused).
 *   Same workspace and argument rules as h3b_blocks_forward; x_save and delta
 *   16-byte aligned (H3B_ERR_ALIGN), owned by the caller; a bad range or a
 *   NULL delta / x_save where needed is H3B_ERR_ARG, checked before anything
 *   else. delta must come from a fresh call with the same dimensions.
 *   h3b_range_delta / h3b_range_apply: the two steps alone, on n elements
 *   (n % 8 == 0, 16-byte aligned). */
H3B_API h3b_status h3b_blocks_forward_cached(const h3b_dims* dims, const h3b_block_weights* w, int n_blocks,
                                             int first, int last, int fresh, const float* c, void* x,
                                             void* x_save, float* delta, void* ws, size_t ws_bytes,
                                             h3b_stream stream);
H3B_API h3b_status h3b_range_delta(const void* before, const void* after, float* delta, long long n,
                                   h3b_stream stream);
H3B_API h3b_status h3b_range_apply(void* x, const float* delta, long long n, h3b_stream stream);

/* CUDA Graph of a multi-block pass: h3b_graph_capture_blocks records
 * h3b_blocks_forward(dims, w, n_blocks, c, x, ws, ws_bytes) (every launch, with
 * its arguments) without running it; h3b_graph_launch replays the whole pass on
 * `stream` as one graph launch. The result is that of h3b_blocks_forward with
 * the same arguments (same kernels); only the per-launch host cost and the gaps
 * between launches go away.
 *   Ownership: the graph handle belongs to the caller (h3b_graph_destroy). The
 *   graph refers to x, c, the weights and the workspace by address; they must
 *   stay allocated and unmoved while the graph is used, and every replay reads
 *   x as it is when the replay runs.
 *   Errors: the same argument checks as h3b_blocks_forward (nothing is
 *   captured then); H3B_ERR_ARG if profiling is on (h3b_profile_enable) or on
 *   launch from another device than the capture's; H3B_ERR_CUDA on a failed
 *   capture or instantiation. Run the pass once with the same dimensions before
 *   capturing, so that every kernel is loaded.
 *   h3b_graph_kernel_count: kernel launches in one replay (0 for NULL). */
typedef struct h3b_graph_s* h3b_graph;
H3B_API h3b_status h3b_graph_capture_blocks(const h3b_dims* dims, const h3b_block_weights* w, int n_blocks,
                                            const float* c, void* x, void* ws, size_t ws_bytes, h3b_graph* out);
H3B_API h3b_status h3b_graph_launch(h3b_graph g, h3b_stream stream);
H3B_API int h3b_graph_kernel_count(h3b_graph g);
H3B_API void h3b_graph_destroy(h3b_graph g);

/* Token reduction ("h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론",
 * section "속도 및 품질 트레이드오프", the control table's Token Reduction row):
 * horizontally adjacent tokens w = 2k, 2k+1 of each (t, h) row are merged by
 * their mean.
 *   full: dims of the UNMERGED grid (W even); only B, T, H, W and d are read:
 *   d % 8 == 0, d <= 65536, B*T*H*W < 2^31 (H3B_ERR_SHAPE otherwise).
 *   x  bf16 [B][T][H][W][d] -> xm bf16 [B][T][H][W/2][d], xm = bf16((a+b)/2).
 *   xm_copy: optional second destination receiving the same merged tokens
 *   (e.g. the buffer the block then updates in place), or NULL. */
H3B_API h3b_status h3b_token_pair(const h3b_dims* full, const void* x, void* xm, void* xm_copy,
                          h3b_stream stream);

/* out[t,h,2k+j] = bf16(x[t,h,2k+j] + (ym[t,h,k] - xm[t,h,k])), j in {0,1}:
 * the block's delta on each merged token is added at both of its positions of
 * the unmerged residual. out may alias x. xm may be NULL: the merged input is
 * then recomputed from x by the rule of h3b_token_pair (the same bits), which
 * saves reading it. */
H3B_API h3b_status h3b_token_unpair(const h3b_dims* full, const void* x, const void* xm, const void* ym,
                            void* out, h3b_stream stream);

/* Per-output-channel weight quantization (offline; [BLOG] "int8 이 뭔가요": one F32
 * scale per output channel): w fp32 [rows][cols] ->
 * q int8 [rows][cols], s fp32 [rows]; s = absmax/127 (float),
 * q = clamp(round-half-even(w/s), -127, 127); an all-zero row gives s = 0,
 * q = 0. cols % 16 == 0. */
H3B_API h3b_status h3b_quantize_weights(const float* w, int rows, int cols, int8_t* q, float* s,
                                h3b_stream stream);

/* Reads (and optionally clears) the device error word of the current device.
 * Synchronizes the device. *code == 0 means no bounded wait ran out. Bits:
 * 1 << 0..3 a bounded wait ran out (TMA tile, tensor-core commit, epilogue or
 * softmax, drain after an abort), 1 << 4 bad launch parameters, 1 << 5 the
 * test wait of h3b_test_bounded_wait, 1 << 6 (checked build only) an index fell
 * outside its buffer and the access was skipped. */
H3B_API h3b_status h3b_device_error(unsigned int* code, int clear);

/* 1 when this library is the checked build (libh3b_checked.so): every kernel
 * tests the global-memory indices it computes against its buffers' extents
 * before the access, records a miss as 1 << 6 in the device error word and
 * skips that access. It stands in for a memory checker where none can run;
 * the normal build (0) compiles the tests out. */
H3B_API int h3b_checked_build(void);

/* Test hook for failure detection without a GPU fault: one thread on the
 * current device waits, with the bounded wait every pipeline of this library
 * uses, on an mbarrier phase that nothing completes. The wait gives up after
 * limit_ns (1 us to 1 s), ORs 1 << 5 into the device error word and the kernel
 * returns normally; the context stays usable. Synchronous (legacy default
 * stream). *waited_out = 1 when the wait ran out (the expected outcome). */
H3B_API h3b_status h3b_test_bounded_wait(unsigned long long limit_ns, int* waited_out);

/* ---------------------------------------------------------------------------
 * Kernel-level timing. While enabled (per process), every kernel launched by
 * the block entry points (h3b_block_forward, h3b_blocks_forward,
 * h3b_token_pair, h3b_token_unpair) is bracketed by CUDA events recorded on
 * the launch stream. h3b_profile_read synchronizes those events and returns,
 * per kernel name, the launch count and the summed device time in ms; it
 * then clears the record. Returns the number of kernel names written (at most
 * max_entries), or a negative h3b_status.
 * ------------------------------------------------------------------------- */
typedef struct {
  const char* name; /* static string owned by the library */
  int launches;
  double total_ms;
} h3b_kernel_time;

H3B_API h3b_status h3b_profile_enable(int enable);
H3B_API int h3b_profile_read(h3b_kernel_time* out, int max_entries);

/* ---------------------------------------------------------------------------
 * Step entry points. Each runs one step of the block on caller buffers; the
 * block entry points above chain exactly these kernels. They exist so every
 * step can be checked on its own.
 * ------------------------------------------------------------------------- */

/* AdaLN Linear ([README] "Int8 양자화", gated AdaLN; [MLX] "性能上限"):
 * mod[b][j] = sum_k w_ada[j][k] c[b][k] + b_ada[j]; mod fp32 [B][6d]. */
H3B_API h3b_status h3b_adaln_modulation(const h3b_dims* dims, const void* w_ada, const float* b_ada,
                                const float* c, float* mod, h3b_stream stream);

/* Fused LayerNorm + modulation + per-row int8 quantization ([README] "Int8 양자화":
 * the activation quantizer fused into the AdaLN kernel; [BLOG] "int8 이 뭔가요": one
 * F32 scale per row, computed at run time) over rows of x (bf16 [rows][d]); shift/scale fp32 [d] broadcast over rows_per_item rows,
 * then advance by mod_stride floats per batch item (rows_per_item = L,
 * mod_stride = 6d when reading a mod buffer; rows_per_item = rows for one set).
 *   h = bf16(LN(x)(1+scale)+shift); s = absmax(h)/127; q = rint(h/s)
 * q int8 [rows][d], s fp32 [rows]; h_out bf16 [rows][d] or NULL (writes h);
 * absmax_zero: fp32 [rows] set to 0, or NULL. write_codes = 0 skips q/s. */
H3B_API h3b_status h3b_ln_modulate_quantize(const void* x, int rows, int d, float eps, const float* shift,
                                    const float* scale, int rows_per_item, int mod_stride,
                                    int8_t* q, float* s, void* h_out, float* absmax_zero,
                                    int write_codes, h3b_stream stream);

/* Per-row int8 quantization of bf16 rows ([BLOG] "int8 이 뭔가요"; the same rule as
 * the fused kernel) (h bf16 [rows][cols]). If absmax is
 * non-NULL it holds each row's max |h| (as produced by the attention and GELU
 * steps) and the row is read once; otherwise it is computed here. */
H3B_API h3b_status h3b_quantize_rows(const void* h, int rows, int cols, const float* absmax, int8_t* q,
                             float* s, h3b_stream stream);

/* int8 GEMM on tensor cores ([README] "Int8 양자화": int8 projections),
 * C[m][n] = sum_k A[m][k] W[n][k] (exact int32).
 * A int8 [M][K], W int8 [N][K], C int32 [M][N]; M >= 0, N and K positive multiples of 16;
 * M*N, M*K and N*K at most 2^40 (the same rules for every GEMM entry point). */
H3B_API h3b_status h3b_gemm_i8_s32(const int8_t* A, const int8_t* W, int32_t* C, int M, int N, int K,
                           h3b_stream stream);

/* int8 GEMM with dequantizing epilogue: out bf16 [M][N] = bf16(C*sA[m]*sW[n] + bias[n]). */
H3B_API h3b_status h3b_gemm_i8_dequant(const int8_t* A, const float* sA, const int8_t* W, const float* sW,
                               const float* bias, void* out, int M, int N, int K,
                               h3b_stream stream);

/* QKV projection with 3D RoPE ([MLX] "性能上限": RoPE folded ahead of the
 * attention), written head-major ([README] "Metal 4 및 TensorOps"):
 *   qkv bf16 [3][B][n_heads][L][head_dim] (part, batch item, head, token, lane).
 * int8 (dims->qkv_int8 == 1): A int8 [B*L][d] + sA, w->wqkv + w->sqkv.
 * bf16 (dims->qkv_int8 == 0): A bf16 [B*L][d] (sA ignored), w->wqkv_bf16.
 * rope_ws: device scratch of at least h3b_rope_table_bytes(dims) bytes. */
H3B_API h3b_status h3b_qkv_projection(const h3b_dims* dims, const void* A, const float* sA,
                              const h3b_block_weights* w, void* qkv, void* rope_ws,
                              h3b_stream stream);
H3B_API size_t h3b_rope_table_bytes(const h3b_dims* dims);

/* Non-causal attention per batch item and head on the head-major qkv buffer
 * (full attention over all latent tokens: [BLOG] "★ 긴 영상은 나눠 찍는 게 훨씬
 * 쌉니다", step time growing about as frames^1.9).
 * o bf16 [B][L][d] (token-major, head h at columns [h*head_dim, (h+1)*head_dim));
 * absmax fp32 [B*L]: each row's max |o| is max-combined into it (zero it first).
 * Reads B, T, H, W, n_heads and head_dim only: B*n_heads <= 65535, B*L < 2^31. */
H3B_API h3b_status h3b_attention(const h3b_dims* dims, const void* qkv, void* o, float* absmax,
                         h3b_stream stream);

/* int8 GEMM with gated residual epilogue ([README] "Int8 양자화", gated AdaLN),
 * in place on x bf16 [M][N]:
 *   x[m][n] = bf16(x[m][n] + gate[m / rows_per_item][n] * (C*sA[m]*sW[n] + bias[n]))
 * gate fp32, rows of gate_stride floats per batch item. */
H3B_API h3b_status h3b_gemm_i8_gated_residual(const int8_t* A, const float* sA, const int8_t* W,
                                      const float* sW, const float* bias, const float* gate,
                                      int rows_per_item, int gate_stride, void* x, int M, int N,
                                      int K, h3b_stream stream);

/* bf16 GEMM with gated residual epilogue ([README] "Metal 4 및 TensorOps": the BF16
 * attention-output projection), in place on x bf16 [M][N]:
 *   x[m][n] = bf16(x[m][n] + gate[m / rows_per_item][n] * (sum_k A[m][k] W[n][k] + bias[n]))
 * A bf16 [M][K], W bf16 [N][K] (fp32 accumulation); gate as above. The output
 * projection of the block when dims->wo_bf16 == 1. Same argument rules as
 * h3b_gemm_i8_gated_residual (N, K positive multiples of 16; 16-byte aligned
 * pointers). */
H3B_API h3b_status h3b_gemm_bf16_gated_residual(const void* A, const void* W, const float* bias,
                                                const float* gate, int rows_per_item, int gate_stride,
                                                void* x, int M, int N, int K, h3b_stream stream);

/* int8 GEMM with GELU epilogue ([README] "Int8 양자화": int8 MLP): g bf16 [M][N] = bf16(GELU_tanh(C*sA[m]*sW[n] + bias[n]));
 * absmax fp32 [M] max-combined with each row's max |g| (zero it first). */
H3B_API h3b_status h3b_gemm_i8_gelu(const int8_t* A, const float* sA, const int8_t* W, const float* sW,
                            const float* bias, void* g, float* absmax, int M, int N, int K,
                            h3b_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* H3B_H */
