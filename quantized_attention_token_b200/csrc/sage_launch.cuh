// sage_launch.cuh -- kernel parameter blocks and launchers shared by the
// libsage CUDA translation units (pre-pass, attention, C ABI).
#pragma once

#include <cuda.h>   // CUtensorMap (encoded through the runtime's driver entry point)

#include "sage.h"
#include "sage_common.cuh"

namespace sage {

// One pre-pass job (its launches): which tensors to quantize, where they
// are, and the workspace regions it fills.
struct PrepassJob {
  const uint16_t* q = nullptr;
  const uint16_t* k = nullptr;
  const uint16_t* v = nullptr;
  Strides sq{}, sk{}, sv{};
  Seqs seqs;
  int nseq = 0, Hq = 0, Hkv = 0, group = 1;
  int bf16 = 0, gran = 0, smooth_k = 0, smooth_q = 0, pv8 = 1, smooth_v = 0;
  int do_q = 0, do_k = 0, do_v = 0;
  int tiles_q = 0, tiles_k = 0;    // workspace tiles per head
  int one_pass = 0;                // debug: K / V through the cluster kernel where a head fits one
  uint32_t* err = nullptr;
  unsigned long long* k_stat = nullptr;   // [nseq][Hkv][D] int64 (fp16) / fp64 bits (bf16) channel sums
  uint32_t* v_stat = nullptr;             // [nseq][Hkv][D][2]: float bits of channel |max|;
                                          // smooth V: keys of the max and of the negated min
  unsigned long long* v_sum = nullptr;    // [nseq][Hkv][D] channel sums of V (smooth V), like k_stat
  float* v_mean = nullptr;                // [nseq][Hkv][D] (smooth V)
  float* k_mean = nullptr;                // [nseq][Hkv][D]
  float* v_scale = nullptr;               // [nseq][Hkv][D]
  int8_t* q_codes = nullptr;
  float* q_scale = nullptr;               // [Hq][tiles_q][128] (group g of a tile at [g])
  int8_t* k_codes = nullptr;
  float* k_scale = nullptr;               // [Hkv][tiles_k][16]
  uint8_t* v_codes = nullptr;
  float* q_mean = nullptr;                // [Hq][tiles_q][D] (smooth Q)
  float* q_bias = nullptr;                // [Hq][tiles_q][tps*128] smooth-Q score correction (dense)
};

struct AttnParams {
  // 1: the epilogue stores each warp's staged rows with asynchronous bulk
  // tensor stores through the output tensor map (a separate kernel parameter:
  // dense one-level modes); 0: plain stores (varlen, two-level modes, or no
  // encoder available).
  int use_out_map;
  const int8_t* q_codes;
  const float* q_scale;
  const int8_t* k_codes;
  const float* k_scale;
  const uint8_t* v_codes;
  const float* v_scale;
  const float* v_mean;       // smooth V: per-channel mean added to the output, else null
  uint32_t* err;
  Seqs seqs;
  int Hq, Hkv, group;
  int tiles_q, tiles_k;      // workspace tiles per head
  void* out;
  Strides os;
  float sl2;                 // sm_scale * log2(e)
  const float* q_bias;       // smooth Q: [Hq][tiles_q][bias_ld] per-key score corrections, else null
  int bias_ld;
  int gran;
  int lazy_tau;              // conditional rescaling: the reference maximum moves only past +tau (0: always)
  int causal;
  int out_bf16;
  int n_pairs, nseq, n_items;  // work items: n_pairs query-tile groups x Hq heads x nseq sequences (set by attn_forward)
  int max_ctas;              // debug: cap on the persistent grid (0: one CTA per SM)
  int dbg_withhold_k;        // debug: CTA 0 skips the copy of this K tile of its ring (-1: none)
};

// P~V accumulation of the attention kernel: one FP32 TMEM accumulator across
// all KV tiles, or a fresh per-tile partial (FP32 or binary16) added into an
// FP32 register accumulator.
enum { kAccOne = 0, kAccTwo = 1, kAccTwoF16 = 2 };

// prepass.cu
// *path (optional): kPrepassOnePass when K / V went through the cluster
// kernel, kPrepassTwoLaunch when through launches A / B, 0 when neither ran.
enum { kPrepassOnePass = 1, kPrepassTwoLaunch = 2 };
cudaError_t prepass_run(const PrepassJob& j, int D, cudaStream_t s, int* path);

// SAGE_OK for cudaSuccess; otherwise records e as the calling thread's last
// CUDA error (sage_last_cuda_error) and returns SAGE_ERR_CUDA.  (api.cu)
sage_status_t cuda_status(cudaError_t e);
cudaError_t prepass_varlen_offsets(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q, int cap_k,
                                   int* toff_q, int* toff_k, uint32_t* err, cudaStream_t s);

// attn_fwd.cu
int attn_tiles_per_cta(int D, bool pv8, bool acc2);
// out_map: the output as a 4-D tensor map (D, S, H, B) of 16-bit values with
// 64 x 32 boxes in the 128-byte swizzle, read when p.use_out_map is 1.
cudaError_t attn_forward(const AttnParams& p, const CUtensorMap& out_map, int D, bool pv8, int acc, int max_len_q,
                         int nseq, cudaStream_t s);
cudaError_t debug_qk_tile(const int8_t* qt, const int8_t* kt, int D, int32_t* out, uint32_t* err,
                          cudaStream_t s);

}  // namespace sage
