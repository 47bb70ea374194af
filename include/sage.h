/*
 * sage.h -- C ABI of the B200 (sm_100a) quantized attention library (libsage).
 *
 * The library computes SageAttention-style quantized attention forward:
 *   out = softmax(Q K^T * sm_scale [+ causal mask]) V
 * with K smoothed by its per-channel token mean, Q and K quantized to INT8
 * (QK^T on INT8 tensor cores, int32 accumulation), FlashAttention-style online
 * softmax over 128-key tiles, P~ quantized to FP8 E4M3 with a static scale and
 * V to FP8 E4M3 per channel (P~V on FP8 tensor cores), or P~ and V kept in
 * 16 bits.  Sources for the method:
 *   - "SageAttention2" paper summary (sgqg.cn/news/89714), section
 *     SageAttention2方法: smooth Q, per-thread quantization, FP8 P~V with a
 *     static P~ scale and per-channel V scale, FP32 buffer for the PV sums;
 *     section 相关工作: SageAttention quantizes Q/K to INT8 after smoothing K
 *     inside FlashAttention's tiling.
 *   - "Kairos的注意力加速利器SageAttention INT8/FP8量化内核..." (mhpq.cn),
 *     section 二 2.1 (kernel table: INT8 QK^T with FP16 or FP8 PV, fp32 and
 *     fp32+fp32 accumulation, per_warp granularity) and 2.2.
 *   - "SageAttention量化加速框架完整指南" (mhpq.cn), section 五分钟跑通
 *     (sageattn(q, k, v, tensor_layout="HND"|"NHD", is_causal); output has
 *     q's shape), section 性能调优实战 (pv_accum_dtype), section 换进真实模型
 *     (no attention mask), section 最容易踩的四个安装坑 (an unsupported GPU
 *     architecture is an error).
 *   - "SageAttention: Thư viện Attention lượng tử hóa" (topgit.dev), section
 *     Tính năng chính: variable-length batches (sageattn_varlen) and native
 *     grouped-query attention.
 *
 * Conventions for every entry point:
 *   - Pointers named q, k, v, out, ws, cu_seqlens_* are DEVICE pointers of
 *     the current CUDA device; the caller owns all memory.  The library never
 *     allocates or frees device memory.  q, k, v, out must be 16-byte aligned;
 *     ws must be 256-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it; no entry point
 *     synchronizes except sage_get_device_error.
 *   - Argument errors are reported synchronously and nothing is launched.
 *     A CUDA launch error is reported as SAGE_ERR_CUDA.
 *   - Device-side timeouts (a pipeline wait that never completes) never hang:
 *     the kernel records the failure in the workspace's error word, releases
 *     its resources and returns; sage_get_device_error reports it.
 *   - Element (b, h, s, d) of a dense tensor lives at
 *       HND: ((b*H + h)*S + s)*D + d        NHD: ((b*S + s)*H + h)*D + d
 *     and of a packed variable-length tensor at (t*H + h)*D + d with
 *     t = cu_seqlens[b] + s.  out has q's layout and dtype.
 *   - D (head dim) is 64 or 128.  Hq % Hkv == 0; query head h reads KV head
 *     h / (Hq / Hkv).  sm_scale <= 0 selects 1/sqrt(D).
 *   - Only NVIDIA B200-class devices (compute capability 10.0) are supported;
 *     any other device gives SAGE_ERR_UNSUPPORTED.
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad enum, misalignment */
  SAGE_ERR_UNSUPPORTED = 2,  /* device is not sm_100, D not in {64,128}, ... */
  SAGE_ERR_WORKSPACE = 3,    /* ws_bytes smaller than the planner's figure */
  SAGE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  SAGE_ERR_TIMEOUT = 5       /* a device pipeline wait gave up (see above) */
} sage_status_t;

typedef enum { SAGE_HND = 0, SAGE_NHD = 1 } sage_layout_t;
typedef enum { SAGE_F16 = 0, SAGE_BF16 = 1 } sage_dtype_t;

/* Q/K quantization groups (the pages name the granularities but define
 * none).  Tokens are counted from the start of their sequence, in blocks of
 * 128; within a block:
 *   PER_BLOCK : Q one group of 128 rows;  K two groups of 64 rows.
 *   PER_WARP  : Q four groups of 32 rows; K two groups of 64 rows.
 *   PER_THREAD: Q rows of each 32-row slice with equal (row mod 8) share a
 *               scale (32 groups); K rows of each 64-row half with equal
 *               (row mod 8) share a scale (16 groups).
 *   PER_TOKEN : Q one group per row (128 groups) [repo summary, Tinh nang
 *               chinh: per-token granularity]; K two groups of 64 rows.
 * q_scale holds 128 slots per tile, k_scale 16 (unused slots are unwritten). */
typedef enum { SAGE_PER_BLOCK = 0, SAGE_PER_WARP = 1, SAGE_PER_THREAD = 2, SAGE_PER_TOKEN = 3 } sage_gran_t;

/* P~V precision: FP8 E4M3 (P~ scale 1/448 static, V scale per channel) or
 * 16-bit (P~ rounded to the input's 16-bit type, V unquantized).
 * FP8_SMOOTH_V: FP8 with V smoothed first -- V less its per-channel mean over
 * the sequence's tokens is quantized, and the mean is added to the output
 * (softmax rows sum to 1) [SageAttention2 summary, SageAttention2方法: the
 * optional smooth-V step]. */
typedef enum { SAGE_PV_FP8 = 0, SAGE_PV_FP16 = 1, SAGE_PV_FP8_SMOOTH_V = 2 } sage_pv_t;

/* P~V accumulation: FP32 = one FP32 tensor-memory accumulator across all KV
 * tiles; FP32_FP32 = a fresh FP32 partial sum per 128-key tile added into a
 * separate FP32 register accumulator (two-level accumulation).
 * FP32_LAZY = FP32 with conditional rescaling: P~ and O stay relative to a
 * reference maximum that moves only when a tile's maximum exceeds it by more
 * than tau (tau = 2 with FP8 P~V, whose static P~ scale becomes 448 * 2^-2;
 * tau = 8 with 16-bit P~V), so most tiles skip the rescale of O.
 * FP32_FP16 = two-level with a binary16 inner level [Kairos page, section 二
 * 2.1, sm89 row: fp32fp16 two-level accumulation; install/tuning guide,
 * 性能调优实战: pv_accum_dtype]: each 128-key tile's partial sum is held in
 * binary16 by the tensor core and added into the FP32 register accumulator.
 * FP8 P~V only (SAGE_PV_FP16 gives SAGE_ERR_UNSUPPORTED).  P~ is encoded
 * with the static scale 1 instead of 448, the largest that keeps one tile's
 * partial sums (128 keys x P~ <= 1 x V codes <= 448 = 57344) inside
 * binary16's range. */
typedef enum { SAGE_ACC_FP32 = 0, SAGE_ACC_FP32_FP32 = 1, SAGE_ACC_FP32_LAZY = 2,
               SAGE_ACC_FP32_FP16 = 3 } sage_acc_t;

/* ------------------------------------------------------------------------ */
/* Workspace.                                                               */
/* ------------------------------------------------------------------------ */
/* Bytes of device workspace a dense call (B sequences of S tokens) needs.
 * Returns 0 for invalid sizes.  smooth_q adds the smooth-Q regions. */
size_t sage_workspace_bytes(int B, int Hq, int Hkv, int S, int D, sage_pv_t pv, int smooth_q);

/* Bytes for a packed variable-length call: n_seqs sequences with at most
 * total_q / total_k tokens in all and max_seqlen tokens in the longest one. */
size_t sage_varlen_workspace_bytes(int n_seqs, int total_q, int total_k, int max_seqlen,
                                   int Hq, int Hkv, int D, sage_pv_t pv);

/* Byte offsets of the workspace regions (for callers that read the quantized
 * tensors, e.g. to cache K/V).  Quantized tiles hold 128 tokens; tile t of
 * sequence b is global tile tile_off(b) + t (dense: b*ceil(S/128) + t).
 *   q_codes : int8  [Hq ][tiles_q][128 rows][D]   swizzled, see below
 *   q_scale : float [Hq ][tiles_q][128]           group g of the tile at [g]
 *   k_codes : int8  [Hkv][tiles_k][128 rows][D]   swizzled
 *   k_scale : float [Hkv][tiles_k][16]
 *   k_mean  : float [n_seqs][Hkv][D]              (0 when smooth_k is off)
 *   v_codes : [Hkv][tiles_k][D rows][128 keys]    E4M3 (1 byte) or 16-bit
 *             (2 bytes, as two [D][64-key] halves of 128-byte rows)
 *   v_scale : float [n_seqs][Hkv][D]              (FP8 mode)
 *   v_mean  : float [n_seqs][Hkv][D]              (FP8_SMOOTH_V; else unwritten)
 *   q_mean  : float [Hq][tiles_q][D]              (smooth_q)
 *   q_bias  : float [Hq][tiles_q][tiles_k_seq*128] (smooth_q, dense only)
 * Swizzle of every 128-byte row r (D=128 codes, E4M3 V rows, 16-bit V halves):
 * logical 16-byte chunk c is stored at chunk c ^ (r % 8).  For 64-byte rows
 * (D=64 codes): chunk c (of 4) is stored at chunk c ^ ((r / 2) % 4).  This is
 * the 128B / 64B swizzle of the tensor cores' shared-memory operand layout, so
 * a tile is copied to shared memory as one contiguous block. */
typedef struct {
  size_t err;       /* uint32 device error word */
  size_t tile_off_q, tile_off_k;   /* int32 [n_seqs+1] (varlen) */
  size_t k_stat, v_sum, v_stat;    /* pre-pass accumulators */
  size_t k_mean, v_scale, v_mean;
  size_t q_codes, q_scale, k_codes, k_scale, v_codes;
  size_t q_mean, q_bias;
  size_t total;
  int tiles_q, tiles_k;            /* tiles per head */
} sage_ws_layout_t;

sage_status_t sage_workspace_layout(int n_seqs, int total_q, int total_k, int max_seqlen,
                                    int Hq, int Hkv, int D, sage_pv_t pv, int smooth_q,
                                    int varlen, sage_ws_layout_t* out);

/* ------------------------------------------------------------------------ */
/* Pre-pass: smooth + quantize.                                             */
/* ------------------------------------------------------------------------ */
/* Smooth K (per-channel mean over each sequence's tokens, when smooth_k),
 * optionally smooth Q (mean of each 128-token block, when smooth_q), and
 * quantize Q and K to INT8 at granularity `gran` into ws.  [SageAttention2
 * summary, 相关工作 and SageAttention2方法; Kairos page 2.2]
 * Reads q [B,Hq,S,D] / [B,S,Hq,D] and k likewise with Hkv heads (dtype,
 * layout).  Writes ws regions k_stat, k_mean, q_codes, q_scale, k_codes,
 * k_scale (+ q_mean, q_bias when smooth_q). */
sage_status_t sage_quant_qk(const void* q, const void* k, sage_dtype_t dtype, sage_layout_t layout,
                            int B, int Hq, int Hkv, int S, int D, sage_gran_t gran,
                            int smooth_k, int smooth_q, void* ws, size_t ws_bytes, void* stream);

/* The whole pre-pass: sage_quant_qk and sage_quant_v together, in two
 * launches (Q tiles and the K / V statistics, then the K and V tiles) plus,
 * with smooth_q, the launch of the per-key smooth-Q corrections. */
sage_status_t sage_quant_qkv(const void* q, const void* k, const void* v, sage_dtype_t dtype,
                             sage_layout_t layout, int B, int Hq, int Hkv, int S, int D,
                             sage_gran_t gran, sage_pv_t pv, int smooth_k, int smooth_q, void* ws,
                             size_t ws_bytes, void* stream);

/* Quantize V per channel to E4M3 (SAGE_PV_FP8; smoothed first with
 * SAGE_PV_FP8_SMOOTH_V) or re-lay it out in 16 bits (SAGE_PV_FP16),
 * transposed to [D][keys] tiles.  [SageAttention2
 * summary, SageAttention2方法, FP8 quantization of P~V]  Writes v_stat,
 * v_scale, v_codes. */
sage_status_t sage_quant_v(const void* v, sage_dtype_t dtype, sage_layout_t layout, int B, int Hkv,
                           int S, int D, sage_pv_t pv, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Attention.                                                               */
/* ------------------------------------------------------------------------ */
/* The attention kernel runs a persistent grid of one CTA per SM over the
 * problem's work items (two 128-row query tiles, or one in two-level mode,
 * of one sequence and head).  sage_debug_set_max_ctas caps that grid;
 * results do not depend on it. */

/* The whole forward pass: sage_quant_qkv + the attention kernel.  out has q's shape, layout and dtype.  [Install/tuning guide,
 * 五分钟跑通 and 性能调优实战] */
sage_status_t sage_attn_fwd(const void* q, const void* k, const void* v, void* out,
                            sage_dtype_t dtype, int B, int Hq, int Hkv, int S, int D,
                            sage_layout_t layout, int is_causal, float sm_scale,
                            sage_gran_t gran, sage_pv_t pv, sage_acc_t pv_accum,
                            int smooth_k, int smooth_q, void* ws, size_t ws_bytes, void* stream);

/* The attention kernel alone, on a workspace already filled by
 * sage_quant_qk and sage_quant_v for the same problem (lets callers keep
 * quantized K/V; also what the benchmark times as the attention kernel). */
sage_status_t sage_attn_quantized(void* out, sage_dtype_t dtype, int B, int Hq, int Hkv, int S,
                                  int D, sage_layout_t layout, int is_causal, float sm_scale,
                                  sage_gran_t gran, sage_pv_t pv, sage_acc_t pv_accum,
                                  int smooth_q, const void* ws, size_t ws_bytes, void* stream);

/* Packed variable-length batch with grouped-query attention [repo summary,
 * Tính năng chính].  q [total_q, Hq, D], k/v [total_k, Hkv, D], out like q.
 * cu_seqlens_q/k: device int32 [n_seqs+1], non-decreasing, starting at 0;
 * sequence b holds tokens [cu[b], cu[b+1]).  max_seqlen bounds every
 * sequence's length (larger lengths are an error reported through the device
 * error word).  total_q/total_k are the token counts the buffers hold.
 * Query and key sequences may differ in length (sequence b attends with its
 * queries cu_seqlens_q[b].. to its keys cu_seqlens_k[b]..).  Causal masking
 * is top-left aligned: query i sees key j iff j <= i, both counted from their
 * sequence's start.  A query with no visible key (its sequence has no keys)
 * gets a zero row. */
sage_status_t sage_attn_varlen_fwd(const void* q, const void* k, const void* v, void* out,
                                   sage_dtype_t dtype, const int* cu_seqlens_q,
                                   const int* cu_seqlens_k, int n_seqs, int total_q, int total_k,
                                   int max_seqlen, int Hq, int Hkv, int D, int is_causal,
                                   float sm_scale, sage_gran_t gran, sage_pv_t pv,
                                   sage_acc_t pv_accum, int smooth_k, void* ws, size_t ws_bytes,
                                   void* stream);

/* ------------------------------------------------------------------------ */
/* Allocation-free forward pass.                                            */
/* ------------------------------------------------------------------------ */
/* The pages have no counterpart to this call; it is a convenience of this
 * library for callers that cannot allocate device memory where they run
 * attention -- e.g. a plugin inside an engine that has already reserved the
 * device's memory for its own pool, code held to a fixed memory budget after
 * start-up, or latency-critical code that cannot accept cudaMalloc's implicit
 * device synchronization.
 *
 * Same arguments and result as sage_attn_fwd (without smooth_q and without a
 * workspace).  The workspace is a static device array of
 * SAGE_NOALLOC_SCRATCH_BYTES inside the library: every GPU that loads the
 * library holds it until the process exits.  Problems whose workspace
 * (sage_workspace_bytes) exceeds that size are rejected with
 * SAGE_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - No device memory is allocated or freed, by this call or the library.
 *   - All calls on a device share the one array: calls whose work overlaps on
 *     the GPU (different streams, or different host threads) race and may
 *     produce wrong results.  Serialize them (one stream, or events).
 *   - Device-side timeouts are recorded in the shared array and cleared by
 *     the next call; use sage_attn_fwd with your own workspace to read them
 *     through sage_get_device_error. */
#define SAGE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

sage_status_t sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                    sage_dtype_t dtype, int B, int Hq, int Hkv, int S, int D,
                                    sage_layout_t layout, int is_causal, float sm_scale,
                                    sage_gran_t gran, sage_pv_t pv, sage_acc_t pv_accum,
                                    int smooth_k, void* stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics.                                                             */
/* ------------------------------------------------------------------------ */
/* Synchronizes `stream`, reads and clears the workspace error word.  Returns
 * SAGE_OK, SAGE_ERR_TIMEOUT (a device wait gave up), SAGE_ERR_INVALID_ARG (a
 * device-side argument check failed, e.g. a varlen length above max_seqlen)
 * or SAGE_ERR_CUDA.  *bits (optional) receives the raw error word. */
sage_status_t sage_get_device_error(void* ws, void* stream, uint32_t* bits);

/* The CUDA runtime error (a cudaError_t value) behind the calling thread's
 * most recent SAGE_ERR_CUDA, and its name (e.g. "cudaErrorInvalidValue");
 * 0 / "cudaSuccess" before any.  Not reset by later successful calls.  The
 * name is a static string owned by the CUDA runtime. */
int sage_last_cuda_error(void);
const char* sage_last_cuda_error_name(void);

/* Debug: cap the attention kernel's persistent grid at max_ctas CTAs (0: one
 * CTA per SM, the default).  Process-wide; applies to the attention launches
 * that follow.  Results do not depend on it: the tests use it to make a few
 * CTAs walk many work items.  max_ctas < 0 gives SAGE_ERR_INVALID_ARG. */
sage_status_t sage_debug_set_max_ctas(int max_ctas);

/* Debug: make the attention launches that follow lose one K tile.  The
 * loader of CTA 0 skips the copy of the ring_index-th K tile it would load
 * (counted from 0 over that CTA's work items); the wait for that tile runs
 * out after about 2 s, the kernel tears down and the workspace's error word
 * reports a timeout, which sage_get_device_error returns as
 * SAGE_ERR_TIMEOUT.  This exercises the timeout path without a GPU fault:
 * no copy is left in flight and the CUDA context stays usable.  The output
 * rows of the aborted CTA's work items are undefined.  -1 (the default)
 * switches it off; values below -1 give SAGE_ERR_INVALID_ARG. */
sage_status_t sage_debug_withhold_k_tile(int ring_index);

/* Debug: on = 1 sends K and V of the pre-passes that follow through the
 * one-pass cluster path wherever a head's keys fit the shared memory of one
 * thread-block cluster (up to 16 CTAs x 128 KB): K and V are read from HBM
 * once instead of twice.  0 (the default) keeps the two-launch path
 * (statistics launch, then quantize launch), which measured faster on B200
 * for every workload tried.  Both paths write identical bytes.  Process-wide.
 * Other values give SAGE_ERR_INVALID_ARG. */
sage_status_t sage_debug_set_prepass_one_pass(int on);

/* Debug: the K / V path the calling thread's last pre-pass took: 1 the
 * one-pass cluster path, 2 the two-launch path, 0 none (no K or V, or no
 * pre-pass yet). */
int sage_debug_last_prepass_path(void);

/* Debug: on = 1 (the default) lets dense attention with one-level
 * accumulation (fp32, fp32_lazy) write its output through a tensor map with
 * asynchronous bulk tensor stores of each warp's staged rows; 0 makes every
 * launch write the staged rows with per-warp 16-byte stores, the path that
 * varlen and the two-level modes always take.  Both paths write identical
 * bytes.  Process-wide.  Other values give SAGE_ERR_INVALID_ARG. */
sage_status_t sage_debug_set_out_map(int on);

/* Debug: the output store path of the calling thread's last attention launch:
 * 1 the tensor map, 2 stores from the threads (per-warp rows in one-level
 * modes, each thread's row in two-level modes), 0 none yet. */
int sage_debug_last_out_path(void);

/* Debug: the int32 scores of one 128x128 tile, S = Q_codes(q tile) *
 * K_codes(k tile)^T, computed by the same tensor-core MMA path as the
 * attention kernel from a workspace filled by sage_quant_qk.  s_out: device
 * int32 [128][128] (row = query, column = key).  Dense problems only. */
sage_status_t sage_debug_qk_tile(const void* ws, int B, int Hq, int Hkv, int S, int D,
                                 sage_pv_t pv, int smooth_q, int b, int h, int q_tile, int k_tile,
                                 int32_t* s_out, void* stream);

const char* sage_status_string(sage_status_t s);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_H_ */
