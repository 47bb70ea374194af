// sage_launch.cuh -- kernel parameter blocks and launchers shared by the
// libsage CUDA translation units (pre-pass, attention, C ABI).
#pragma once

#include "sage_common.cuh"

namespace sage {

struct PrepassParams {
  const uint16_t* x;          // input tensor (fp16 / bf16 bits)
  Strides st;
  Seqs seqs;
  int H;                      // heads of this tensor
  int bf16;
  int gran;
  int smooth;                 // K: subtract channel mean; Q: subtract block mean
  int tiles;                  // workspace tiles per head
  uint32_t* err;
  unsigned long long* k_stat; // [nseq][H][D] int64 (fp16) / fp64 bits (bf16) channel sums
  uint32_t* v_stat;           // [nseq][H][D] float bits of channel |max|
  float* k_mean;              // [nseq][H][D]
  float* v_scale;             // [nseq][H][D]
  int8_t* codes;              // Q or K tiles
  float* scales;              // [H][tiles][32 or 16]
  uint8_t* v_codes;           // V tiles
  float* q_mean;              // [H][tiles][D] (smooth Q)
};

struct AttnParams {
  const int8_t* q_codes;
  const float* q_scale;
  const int8_t* k_codes;
  const float* k_scale;
  const uint8_t* v_codes;
  const float* v_scale;
  uint32_t* err;
  Seqs seqs;
  int Hq, Hkv, group;
  int tiles_q, tiles_k;      // workspace tiles per head
  void* out;
  Strides os;
  float sl2;                 // sm_scale * log2(e)
  int gran;
  int causal;
  int out_bf16;
};

// prepass.cu
cudaError_t prepass_qk(const PrepassParams& pq, const PrepassParams& pk, int D, int nseq, int tps_q,
                       int tps_k, cudaStream_t s);
cudaError_t prepass_v(const PrepassParams& pv, int D, bool pv8, int nseq, int tps, cudaStream_t s);
cudaError_t prepass_varlen_offsets(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q,
                                   int cap_k, int* toff_q, int* toff_k, uint32_t* err, cudaStream_t s);

// attn_fwd.cu
int attn_tiles_per_cta(int D, bool pv8, bool acc2);
cudaError_t attn_forward(const AttnParams& p, int D, bool pv8, bool acc2, int max_len_q, int nseq,
                         cudaStream_t s);
cudaError_t debug_qk_tile(const int8_t* qt, const int8_t* kt, int D, int32_t* out, uint32_t* err,
                          cudaStream_t s);

}  // namespace sage
