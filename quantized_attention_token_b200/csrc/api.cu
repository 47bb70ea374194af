// api.cu -- the C ABI of libsage (declared in include/sage.h).
//
// Host side only: argument validation, the workspace planner, and the order
// of launches on the caller's stream.  No device memory is allocated here and
// no call synchronizes except sage_get_device_error.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>

#include "sage.h"
#include "sage_launch.cuh"

#define SAGE_EXPORT extern "C" __attribute__((visibility("default")))

namespace sage {

// The CUDA error behind the calling thread's last SAGE_ERR_CUDA.
thread_local int g_last_cuda_error = 0;

sage_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SAGE_OK;
  g_last_cuda_error = (int)e;
  return SAGE_ERR_CUDA;
}

namespace {

// Debug settings (sage_debug_set_max_ctas, sage_debug_withhold_k_tile,
// sage_debug_set_prepass_one_pass, sage_debug_set_out_map): process-wide, read
// at each launch.
std::atomic<int> g_max_ctas{0};
std::atomic<int> g_withhold_k{-1};
std::atomic<int> g_prepass_one_pass{0};
std::atomic<int> g_out_map{1};
// The K / V path of the calling thread's last pre-pass (kPrepassOnePass /
// kPrepassTwoLaunch, 0 none).
thread_local int g_last_prepass_path = 0;
// The output store path of the calling thread's last attention launch
// (1 tensor map, 2 stores from the threads, 0 none).
thread_local int g_last_out_path = 0;

// ---------------------------------------------------------------- device check
sage_status_t check_device() {
  static int cache[128] = {0};   // 0 unknown, 1 sm_100, -1 other
  int dev = 0;
  if (sage_status_t st = cuda_status(cudaGetDevice(&dev))) return st;
  if (dev < 0 || dev >= 128) return SAGE_ERR_UNSUPPORTED;
  if (cache[dev] == 0) {
    int maj = 0, mnr = 0;
    if (sage_status_t st = cuda_status(cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev))) return st;
    if (sage_status_t st = cuda_status(cudaDeviceGetAttribute(&mnr, cudaDevAttrComputeCapabilityMinor, dev))) return st;
    cache[dev] = (maj == 10 && mnr == 0) ? 1 : -1;
  }
  return cache[dev] == 1 ? SAGE_OK : SAGE_ERR_UNSUPPORTED;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
size_t up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int cdiv(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- planner
// Regions in order: error word, varlen tile offsets, K/V statistics, K/V
// results, then the Q results (so the K/V part does not depend on Hq).
sage_status_t plan(int nseq, int total_q, int total_k, int max_seqlen, int Hq, int Hkv, int D, int pv,
                   int smooth_q, int varlen, sage_ws_layout_t* L) {
  if (nseq <= 0 || max_seqlen <= 0 || Hq <= 0 || Hkv <= 0 || total_q < 0 || total_k < 0)
    return SAGE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return SAGE_ERR_UNSUPPORTED;
  if (pv != SAGE_PV_FP8 && pv != SAGE_PV_FP16 && pv != SAGE_PV_FP8_SMOOTH_V) return SAGE_ERR_INVALID_ARG;
  if (smooth_q && varlen) return SAGE_ERR_UNSUPPORTED;
  if (max_seqlen > (1 << 24) || nseq > (1 << 20) || Hq > 4096) return SAGE_ERR_UNSUPPORTED;
  const long long tps = cdiv(max_seqlen, kTile);
  const long long tq = varlen ? (long long)total_q / kTile + nseq : (long long)nseq * tps;
  const long long tk = varlen ? (long long)total_k / kTile + nseq : (long long)nseq * tps;
  if (tq > INT_MAX / 2 || tk > INT_MAX / 2) return SAGE_ERR_UNSUPPORTED;
  std::memset(L, 0, sizeof(*L));
  L->tiles_q = (int)tq;
  L->tiles_k = (int)tk;
  size_t o = 0;
  auto take = [&](size_t bytes, size_t align) { o = up(o, align); size_t r = o; o += bytes; return r; };
  const size_t nd = (size_t)nseq * Hkv * D;
  L->err = take(256, 256);
  L->tile_off_q = take(varlen ? sizeof(int) * (nseq + 1) : 0, 256);
  L->tile_off_k = take(varlen ? sizeof(int) * (nseq + 1) : 0, 256);
  // k_stat, v_sum and v_stat are contiguous: one memset zeroes them before
  // each pre-pass.  v_stat: per channel two uint32 (|max| bits; smooth V:
  // order-preserving keys of the maximum and of the negated minimum).
  L->k_stat = take(nd * 8, 256);
  L->v_sum = take(nd * 8, 8);
  L->v_stat = take(nd * 8, 8);
  L->k_mean = take(nd * 4, 256);
  L->v_scale = take(nd * 4, 256);
  L->v_mean = take(nd * 4, 256);
  L->k_codes = take((size_t)Hkv * tk * kTile * D, 1024);
  L->k_scale = take((size_t)Hkv * tk * kKGroupsMax * 4, 256);
  // sized for 16-bit V in both modes, so every region's offset is the same
  // whichever P~V precision a later call picks
  L->v_codes = take((size_t)Hkv * tk * kTile * D * 2, 1024);
  L->q_codes = take((size_t)Hq * tq * kTile * D, 1024);
  L->q_scale = take((size_t)Hq * tq * kQGroupsMax * 4, 256);
  L->q_mean = take(smooth_q ? (size_t)Hq * tq * D * 4 : 0, 256);
  L->q_bias = take(smooth_q ? (size_t)Hq * tq * tps * kTile * 4 : 0, 256);
  L->total = up(o, 256);
  return SAGE_OK;
}

template <class T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off); }

Strides dense_strides(sage_layout_t layout, int H, int S, int D) {
  if (layout == SAGE_HND) return Strides{(long long)H * S * D, (long long)S * D, (long long)D};
  return Strides{(long long)S * H * D, (long long)D, (long long)H * D};
}


sage_status_t check_common(sage_dtype_t dtype, int D, sage_gran_t gran, sage_pv_t pv, sage_acc_t acc) {
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return SAGE_ERR_INVALID_ARG;
  if (gran != SAGE_PER_BLOCK && gran != SAGE_PER_WARP && gran != SAGE_PER_THREAD && gran != SAGE_PER_TOKEN)
    return SAGE_ERR_INVALID_ARG;
  if (pv != SAGE_PV_FP8 && pv != SAGE_PV_FP16 && pv != SAGE_PV_FP8_SMOOTH_V) return SAGE_ERR_INVALID_ARG;
  if (acc != SAGE_ACC_FP32 && acc != SAGE_ACC_FP32_FP32 && acc != SAGE_ACC_FP32_LAZY && acc != SAGE_ACC_FP32_FP16)
    return SAGE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  // the binary16 inner accumulation is defined for FP8 P~V (its P~ scale keeps
  // one tile's partial sums inside binary16's range)
  if (acc == SAGE_ACC_FP32_FP16 && pv == SAGE_PV_FP16) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

// Bytes of the pre-pass accumulators k_stat .. v_stat (zeroed per pre-pass).
size_t stats_zero_bytes(const sage_ws_layout_t& L, int nseq, int Hkv, int D) {
  return L.v_stat + 8 * (size_t)nseq * Hkv * D - L.k_stat;
}

// The pre-pass over any of Q, K, V (dense or varlen).
sage_status_t run_prepass(const void* q, const void* k, const void* v, int bf16, Strides sq, Strides sk,
                          Strides sv, const Seqs& seqs, int nseq, int Hq, int Hkv, int D, int gran, int pv,
                          int smooth_k, int smooth_q, void* ws, const sage_ws_layout_t& L, cudaStream_t s) {
  if (sage_status_t st = cuda_status(cudaMemsetAsync(at<char>(ws, L.k_stat), 0, stats_zero_bytes(L, nseq, Hkv, D), s)))
    return st;
  if (seqs.cu_k) {
    // A varlen sequence without keys gets no K / V tile, so nothing else
    // writes its K means and V scales / means: zero them, so that its queries
    // (no visible key: output 0) read zeros rather than stale workspace bytes.
    const size_t nd = (size_t)nseq * Hkv * D;
    if (k)
      if (sage_status_t st = cuda_status(cudaMemsetAsync(at<char>(ws, L.k_mean), 0, nd * 4, s))) return st;
    if (v)
      if (sage_status_t st = cuda_status(cudaMemsetAsync(at<char>(ws, L.v_scale), 0, L.v_mean + nd * 4 - L.v_scale, s)))
        return st;
  }
  PrepassJob j;
  j.q = static_cast<const uint16_t*>(q);
  j.k = static_cast<const uint16_t*>(k);
  j.v = static_cast<const uint16_t*>(v);
  j.sq = sq;
  j.sk = sk;
  j.sv = sv;
  j.seqs = seqs;
  j.nseq = nseq;
  j.Hq = Hq;
  j.Hkv = Hkv;
  j.group = Hq / Hkv;
  j.bf16 = bf16;
  j.gran = gran;
  j.smooth_k = smooth_k ? 1 : 0;
  j.smooth_q = smooth_q ? 1 : 0;
  j.pv8 = pv != SAGE_PV_FP16;
  j.smooth_v = pv == SAGE_PV_FP8_SMOOTH_V;
  j.do_q = q != nullptr;
  j.do_k = k != nullptr;
  j.do_v = v != nullptr;
  j.tiles_q = L.tiles_q;
  j.tiles_k = L.tiles_k;
  j.err = at<uint32_t>(ws, L.err);
  j.k_stat = at<unsigned long long>(ws, L.k_stat);
  j.v_stat = at<uint32_t>(ws, L.v_stat);
  j.v_sum = at<unsigned long long>(ws, L.v_sum);
  j.v_mean = at<float>(ws, L.v_mean);
  j.k_mean = at<float>(ws, L.k_mean);
  j.v_scale = at<float>(ws, L.v_scale);
  j.q_codes = at<int8_t>(ws, L.q_codes);
  j.q_scale = at<float>(ws, L.q_scale);
  j.k_codes = at<int8_t>(ws, L.k_codes);
  j.k_scale = at<float>(ws, L.k_scale);
  j.v_codes = at<uint8_t>(ws, L.v_codes);
  j.q_mean = smooth_q ? at<float>(ws, L.q_mean) : nullptr;
  j.q_bias = smooth_q ? at<float>(ws, L.q_bias) : nullptr;
  if (seqs.cu_k)
    if (sage_status_t st = cuda_status(prepass_varlen_offsets(seqs.cu_q, seqs.cu_k, nseq, seqs.max_seqlen, L.tiles_q,
                                                              L.tiles_k, const_cast<int*>(seqs.toff_q),
                                                              const_cast<int*>(seqs.toff_k), j.err, s)))
      return st;
  j.one_pass = g_prepass_one_pass.load();
  return cuda_status(prepass_run(j, D, s, &g_last_prepass_path));
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link to the
// driver library); null when the driver does not provide it.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      (void)cudaGetLastError();
      return (EncodeTiledFn) nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// The output as a 4-D tensor (D, S, H, B) of 16-bit values (HND and NHD differ
// only in the strides), boxes of 64 columns x 32 rows, 128-byte swizzle.  Rows
// past S fall outside the tensor, so the stores clip the last tile.  False
// (plain stores) when the encoder is missing or refuses the shape.
bool encode_out_map(CUtensorMap& m, const AttnParams& p, int D, int B, int H, int S) {
  const EncodeTiledFn enc = encode_tiled();
  if (!enc || S <= 0) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)p.os.ss * 2, (cuuint64_t)p.os.sh * 2, (cuuint64_t)p.os.sb * 2};
  const cuuint32_t box[4] = {64, 32, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, p.out, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

sage_status_t run_attn(void* out, int bf16, Strides so, const Seqs& seqs, int nseq, int Hq, int Hkv, int D,
                       int causal, float sm_scale, int gran, int pv, int acc, int smooth_q, const void* ws,
                       const sage_ws_layout_t& L, cudaStream_t s) {
  void* w = const_cast<void*>(ws);
  AttnParams p{};
  p.q_codes = at<int8_t>(w, L.q_codes);
  p.q_scale = at<float>(w, L.q_scale);
  p.k_codes = at<int8_t>(w, L.k_codes);
  p.k_scale = at<float>(w, L.k_scale);
  p.v_codes = at<uint8_t>(w, L.v_codes);
  p.v_scale = at<float>(w, L.v_scale);
  p.err = at<uint32_t>(w, L.err);
  p.seqs = seqs;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.tiles_q = L.tiles_q;
  p.tiles_k = L.tiles_k;
  p.out = out;
  p.os = so;
  const float scale = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf((float)D);
  p.sl2 = scale * kLog2e;
  p.q_bias = smooth_q ? at<float>(w, L.q_bias) : nullptr;
  p.bias_ld = seqs.tps * kTile;
  p.gran = gran;
  p.lazy_tau = acc == SAGE_ACC_FP32_LAZY ? (pv == SAGE_PV_FP16 ? 8 : 2) : 0;
  p.causal = causal ? 1 : 0;
  p.out_bf16 = bf16;
  p.v_mean = pv == SAGE_PV_FP8_SMOOTH_V ? at<float>(w, L.v_mean) : nullptr;
  p.max_ctas = g_max_ctas.load();
  p.dbg_withhold_k = g_withhold_k.load();
  const int mode = acc == SAGE_ACC_FP32_FP32 ? kAccTwo : acc == SAGE_ACC_FP32_FP16 ? kAccTwoF16 : kAccOne;
  // dense one-level: the epilogue stores through a tensor map of the output
  CUtensorMap out_map{};
  p.use_out_map =
      (g_out_map.load() && !seqs.cu_q && mode == kAccOne && encode_out_map(out_map, p, D, nseq, Hq, seqs.S)) ? 1 : 0;
  g_last_out_path = p.use_out_map ? 1 : 2;
  return cuda_status(attn_forward(p, out_map, D, pv != SAGE_PV_FP16, mode, seqs.max_seqlen, nseq, s));
}

Seqs dense_seqs(int S) {
  Seqs q;
  q.S = S;
  q.tps = cdiv(S, kTile);
  q.max_seqlen = S;
  return q;
}

sage_status_t check_dense(int B, int Hq, int Hkv, int S, int D, sage_layout_t layout) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S <= 0) return SAGE_ERR_INVALID_ARG;
  if (layout != SAGE_HND && layout != SAGE_NHD) return SAGE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return SAGE_ERR_UNSUPPORTED;
  if ((long long)B * S * Hq * D > (1ll << 40)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

}  // namespace
}  // namespace sage

using namespace sage;

// ====================================================================== C ABI
SAGE_EXPORT size_t sage_workspace_bytes(int B, int Hq, int Hkv, int S, int D, sage_pv_t pv, int smooth_q) {
  sage_ws_layout_t L;
  if (check_dense(B, Hq, Hkv, S, D, SAGE_HND) != SAGE_OK) return 0;
  if (plan(B, B * S, B * S, S, Hq, Hkv, D, pv, smooth_q, 0, &L) != SAGE_OK) return 0;
  return L.total;
}

SAGE_EXPORT size_t sage_varlen_workspace_bytes(int n_seqs, int total_q, int total_k, int max_seqlen, int Hq,
                                               int Hkv, int D, sage_pv_t pv) {
  sage_ws_layout_t L;
  if (plan(n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv, 0, 1, &L) != SAGE_OK) return 0;
  return L.total;
}

SAGE_EXPORT sage_status_t sage_workspace_layout(int n_seqs, int total_q, int total_k, int max_seqlen, int Hq,
                                                int Hkv, int D, sage_pv_t pv, int smooth_q, int varlen,
                                                sage_ws_layout_t* out) {
  if (!out) return SAGE_ERR_INVALID_ARG;
  return plan(n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv, smooth_q, varlen, out);
}

SAGE_EXPORT sage_status_t sage_quant_qk(const void* q, const void* k, sage_dtype_t dtype, sage_layout_t layout,
                                        int B, int Hq, int Hkv, int S, int D, sage_gran_t gran, int smooth_k,
                                        int smooth_q, void* ws, size_t ws_bytes, void* stream) {
  sage_status_t st;
  if ((st = check_dense(B, Hq, Hkv, S, D, layout)) != SAGE_OK) return st;
  if ((st = check_common(dtype, D, gran, SAGE_PV_FP8, SAGE_ACC_FP32)) != SAGE_OK) return st;
  if (!q || !k || !ws) return SAGE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(ws, 256)) return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  if ((st = plan(B, B * S, B * S, S, Hq, Hkv, D, SAGE_PV_FP8, smooth_q, 0, &L)) != SAGE_OK) return st;
  if (ws_bytes < (smooth_q ? L.total : L.q_scale + (size_t)Hq * L.tiles_q * kQGroupsMax * 4)) return SAGE_ERR_WORKSPACE;
  if ((st = check_device()) != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return run_prepass(q, k, nullptr, dtype == SAGE_BF16, dense_strides(layout, Hq, S, D),
                     dense_strides(layout, Hkv, S, D), Strides{}, dense_seqs(S), B, Hq, Hkv, D, gran, SAGE_PV_FP8,
                     smooth_k, smooth_q, ws, L, s);
}

SAGE_EXPORT sage_status_t sage_quant_v(const void* v, sage_dtype_t dtype, sage_layout_t layout, int B, int Hkv,
                                       int S, int D, sage_pv_t pv, void* ws, size_t ws_bytes, void* stream) {
  sage_status_t st;
  if ((st = check_dense(B, Hkv, Hkv, S, D, layout)) != SAGE_OK) return st;
  if ((st = check_common(dtype, D, SAGE_PER_BLOCK, pv, SAGE_ACC_FP32)) != SAGE_OK) return st;
  if (!v || !ws || !aligned(v, 16) || !aligned(ws, 256)) return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  // the K/V regions do not depend on the number of query heads
  if ((st = plan(B, B * S, B * S, S, Hkv, Hkv, D, pv, 0, 0, &L)) != SAGE_OK) return st;
  if (ws_bytes < L.q_codes) return SAGE_ERR_WORKSPACE;
  if ((st = check_device()) != SAGE_OK) return st;
  return run_prepass(nullptr, nullptr, v, dtype == SAGE_BF16, Strides{}, Strides{}, dense_strides(layout, Hkv, S, D),
                     dense_seqs(S), B, Hkv, Hkv, D, SAGE_PER_BLOCK, pv, 0, 0, ws, L, static_cast<cudaStream_t>(stream));
}

SAGE_EXPORT sage_status_t sage_quant_qkv(const void* q, const void* k, const void* v, sage_dtype_t dtype,
                                         sage_layout_t layout, int B, int Hq, int Hkv, int S, int D, sage_gran_t gran,
                                         sage_pv_t pv, int smooth_k, int smooth_q, void* ws, size_t ws_bytes,
                                         void* stream) {
  sage_status_t st;
  if ((st = check_dense(B, Hq, Hkv, S, D, layout)) != SAGE_OK) return st;
  if ((st = check_common(dtype, D, gran, pv, SAGE_ACC_FP32)) != SAGE_OK) return st;
  if (!q || !k || !v || !ws) return SAGE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(ws, 256)) return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  if ((st = plan(B, B * S, B * S, S, Hq, Hkv, D, pv, smooth_q, 0, &L)) != SAGE_OK) return st;
  if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
  if ((st = check_device()) != SAGE_OK) return st;
  return run_prepass(q, k, v, dtype == SAGE_BF16, dense_strides(layout, Hq, S, D), dense_strides(layout, Hkv, S, D),
                     dense_strides(layout, Hkv, S, D), dense_seqs(S), B, Hq, Hkv, D, gran, pv, smooth_k, smooth_q,
                     ws, L, static_cast<cudaStream_t>(stream));
}

SAGE_EXPORT sage_status_t sage_attn_quantized(void* out, sage_dtype_t dtype, int B, int Hq, int Hkv, int S, int D,
                                              sage_layout_t layout, int is_causal, float sm_scale,
                                              sage_gran_t gran, sage_pv_t pv, sage_acc_t pv_accum, int smooth_q,
                                              const void* ws, size_t ws_bytes, void* stream) {
  sage_status_t st;
  if ((st = check_dense(B, Hq, Hkv, S, D, layout)) != SAGE_OK) return st;
  if ((st = check_common(dtype, D, gran, pv, pv_accum)) != SAGE_OK) return st;
  if (!out || !ws || !aligned(out, 16) || !aligned(ws, 256)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  if ((st = plan(B, B * S, B * S, S, Hq, Hkv, D, pv, smooth_q, 0, &L)) != SAGE_OK) return st;
  if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
  if ((st = check_device()) != SAGE_OK) return st;
  return run_attn(out, dtype == SAGE_BF16, dense_strides(layout, Hq, S, D), dense_seqs(S), B, Hq, Hkv, D,
                  is_causal, sm_scale, gran, pv, pv_accum, smooth_q, ws, L, static_cast<cudaStream_t>(stream));
}

SAGE_EXPORT sage_status_t sage_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                        sage_dtype_t dtype, int B, int Hq, int Hkv, int S, int D,
                                        sage_layout_t layout, int is_causal, float sm_scale, sage_gran_t gran,
                                        sage_pv_t pv, sage_acc_t pv_accum, int smooth_k, int smooth_q, void* ws,
                                        size_t ws_bytes, void* stream) {
  sage_status_t st;
  if ((st = check_dense(B, Hq, Hkv, S, D, layout)) != SAGE_OK) return st;
  if ((st = check_common(dtype, D, gran, pv, pv_accum)) != SAGE_OK) return st;
  if (!q || !k || !v || !out || !ws) return SAGE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(ws, 256))
    return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  if ((st = plan(B, B * S, B * S, S, Hq, Hkv, D, pv, smooth_q, 0, &L)) != SAGE_OK) return st;
  if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
  if ((st = check_device()) != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int bf16 = dtype == SAGE_BF16;
  const Seqs seqs = dense_seqs(S);
  if ((st = run_prepass(q, k, v, bf16, dense_strides(layout, Hq, S, D), dense_strides(layout, Hkv, S, D),
                        dense_strides(layout, Hkv, S, D), seqs, B, Hq, Hkv, D, gran, pv, smooth_k, smooth_q, ws, L,
                        s)) != SAGE_OK)
    return st;
  return run_attn(out, bf16, dense_strides(layout, Hq, S, D), seqs, B, Hq, Hkv, D, is_causal, sm_scale, gran, pv,
                  pv_accum, smooth_q, ws, L, s);
}

SAGE_EXPORT sage_status_t sage_attn_varlen_fwd(const void* q, const void* k, const void* v, void* out,
                                               sage_dtype_t dtype, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                               int n_seqs, int total_q, int total_k, int max_seqlen, int Hq, int Hkv,
                                               int D, int is_causal, float sm_scale, sage_gran_t gran, sage_pv_t pv,
                                               sage_acc_t pv_accum, int smooth_k, void* ws, size_t ws_bytes,
                                               void* stream) {
  sage_status_t st;
  if ((st = check_common(dtype, D, gran, pv, pv_accum)) != SAGE_OK) return st;
  if (n_seqs <= 0 || max_seqlen <= 0 || total_q <= 0 || total_k <= 0 || Hq <= 0 || Hkv <= 0)
    return SAGE_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SAGE_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !ws || !cu_seqlens_q || !cu_seqlens_k) return SAGE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(ws, 256) ||
      !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  if ((st = plan(n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv, 0, 1, &L)) != SAGE_OK) return st;
  if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
  if ((st = check_device()) != SAGE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Seqs seqs;
  seqs.cu_q = cu_seqlens_q;
  seqs.cu_k = cu_seqlens_k;
  seqs.toff_q = at<int>(ws, L.tile_off_q);
  seqs.toff_k = at<int>(ws, L.tile_off_k);
  seqs.max_seqlen = max_seqlen;
  const int bf16 = dtype == SAGE_BF16;
  const Strides sq{0, (long long)D, (long long)Hq * D}, skv{0, (long long)D, (long long)Hkv * D};
  if ((st = run_prepass(q, k, v, bf16, sq, skv, skv, seqs, n_seqs, Hq, Hkv, D, gran, pv, smooth_k, 0, ws, L, s)) !=
      SAGE_OK)
    return st;
  return run_attn(out, bf16, sq, seqs, n_seqs, Hq, Hkv, D, is_causal, sm_scale, gran, pv, pv_accum, 0, ws, L, s);
}

SAGE_EXPORT sage_status_t sage_get_device_error(void* ws, void* stream, uint32_t* bits) {
  if (!ws || !aligned(ws, 256)) return SAGE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t w = 0;
  if (sage_status_t st = cuda_status(cudaStreamSynchronize(s))) return st;
  if (sage_status_t st = cuda_status(cudaMemcpy(&w, ws, sizeof(w), cudaMemcpyDeviceToHost))) return st;
  if (w)
    if (sage_status_t st = cuda_status(cudaMemset(ws, 0, sizeof(w)))) return st;
  if (bits) *bits = w;
  if (w & (kErrTimeoutLoad | kErrTimeoutMma | kErrTimeoutSoftmax | kErrTimeoutCorr)) return SAGE_ERR_TIMEOUT;
  if (w) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

SAGE_EXPORT sage_status_t sage_debug_qk_tile(const void* ws, int B, int Hq, int Hkv, int S, int D, sage_pv_t pv,
                                             int smooth_q, int b, int h, int q_tile, int k_tile, int32_t* s_out,
                                             void* stream) {
  sage_status_t st;
  if ((st = check_dense(B, Hq, Hkv, S, D, SAGE_HND)) != SAGE_OK) return st;
  if (!ws || !s_out || !aligned(ws, 256) || !aligned(s_out, 16)) return SAGE_ERR_INVALID_ARG;
  const int tps = cdiv(S, kTile);
  if (b < 0 || b >= B || h < 0 || h >= Hq || q_tile < 0 || q_tile >= tps || k_tile < 0 || k_tile >= tps)
    return SAGE_ERR_INVALID_ARG;
  sage_ws_layout_t L;
  if ((st = plan(B, B * S, B * S, S, Hq, Hkv, D, pv, smooth_q, 0, &L)) != SAGE_OK) return st;
  if ((st = check_device()) != SAGE_OK) return st;
  void* w = const_cast<void*>(ws);
  const int hk = h / (Hq / Hkv);
  const int8_t* qt = at<int8_t>(w, L.q_codes) + ((size_t)h * L.tiles_q + (size_t)b * tps + q_tile) * kTile * D;
  const int8_t* kt = at<int8_t>(w, L.k_codes) + ((size_t)hk * L.tiles_k + (size_t)b * tps + k_tile) * kTile * D;
  return cuda_status(debug_qk_tile(qt, kt, D, s_out, at<uint32_t>(w, L.err), static_cast<cudaStream_t>(stream)));
}

SAGE_EXPORT sage_status_t sage_debug_set_max_ctas(int max_ctas) {
  if (max_ctas < 0) return SAGE_ERR_INVALID_ARG;
  g_max_ctas.store(max_ctas);
  return SAGE_OK;
}

SAGE_EXPORT sage_status_t sage_debug_withhold_k_tile(int ring_index) {
  if (ring_index < -1) return SAGE_ERR_INVALID_ARG;
  g_withhold_k.store(ring_index);
  return SAGE_OK;
}

SAGE_EXPORT sage_status_t sage_debug_set_prepass_one_pass(int on) {
  if (on != 0 && on != 1) return SAGE_ERR_INVALID_ARG;
  g_prepass_one_pass.store(on);
  return SAGE_OK;
}

SAGE_EXPORT int sage_debug_last_prepass_path(void) { return g_last_prepass_path; }

SAGE_EXPORT sage_status_t sage_debug_set_out_map(int on) {
  if (on != 0 && on != 1) return SAGE_ERR_INVALID_ARG;
  g_out_map.store(on);
  return SAGE_OK;
}

SAGE_EXPORT int sage_debug_last_out_path(void) { return g_last_out_path; }

SAGE_EXPORT int sage_last_cuda_error(void) { return sage::g_last_cuda_error; }

SAGE_EXPORT const char* sage_last_cuda_error_name(void) {
  return cudaGetErrorName(static_cast<cudaError_t>(sage::g_last_cuda_error));
}

SAGE_EXPORT const char* sage_status_string(sage_status_t s) {
  switch (s) {
    case SAGE_OK: return "ok";
    case SAGE_ERR_INVALID_ARG: return "invalid argument";
    case SAGE_ERR_UNSUPPORTED: return "unsupported (device must be sm_100; D in {64,128}; Hq % Hkv == 0)";
    case SAGE_ERR_WORKSPACE: return "workspace too small";
    case SAGE_ERR_CUDA: return "CUDA error";
    case SAGE_ERR_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}
