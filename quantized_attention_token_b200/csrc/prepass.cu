// prepass.cu -- smooth + quantize pre-pass (HBM-bound).
//
// Method (SageAttention2 summary, sgqg.cn, sections 相关工作 / SageAttention2方法;
// Kairos SageAttention page, section 2.2):
//   * K is smoothed by subtracting its per-channel mean over the sequence's
//     tokens, then Q and K are quantized to INT8 with one scale per group
//     (granularities per_block / per_warp / per_thread, shapes in sage.h):
//       delta = amax/127,  code = clamp(rne(x * (127/amax)), -127, 127)
//     (float32 throughout; 127/amax is one IEEE division per group).
//   * V is quantized per channel to FP8 E4M3 (delta_c = amax_c/448,
//     code = e4m3_rne_satfinite(v * (448/amax_c))), or kept in 16 bits.
// Outputs go straight into the layout the attention kernel's tensor cores
// read: 128-token tiles, rows swizzled as the 128B / 64B shared-memory operand
// layout, so one bulk copy moves a tile into shared memory.  V is written
// transposed ([D][keys]) so that it is the K-major B operand of P~V.
//
// Traffic per (token, head, channel): Q, K, V read (2 B each) and 1 B each
// written (FP8 mode); the K/V statistics pass reads K and V a second time.
#include "sage_launch.cuh"

namespace sage {

// fp16 value times 2^24 as an exact integer (finite inputs).
__device__ __forceinline__ long long f16_fixed24(uint16_t h) {
  int e = (h >> 10) & 0x1F, m = h & 0x3FF;
  long long v = (e == 0) ? (long long)m : ((long long)(m | 0x400) << (e - 1));
  return (h & 0x8000) ? -v : v;
}

__device__ __forceinline__ void unpack8(const uint4& v, int bf16, float (&f)[8]) {
  const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
  for (int u = 0; u < 8; ++u) f[u] = h16_to_f32(h[u], bf16);
}

// ---------------------------------------------------------------- varlen tile offsets
// toff[b] = sum_{b'<b} ceil(L_b'/128); checks lengths against max_seqlen and
// the workspace's tile capacity.
__global__ void varlen_offsets_kernel(const int* cu_q, const int* cu_k, int n, int max_seqlen,
                                      int cap_q, int cap_k, int* toff_q, int* toff_k, uint32_t* err) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int aq = 0, ak = 0;
  bool bad = cu_q[0] != 0 || cu_k[0] != 0;
  for (int b = 0; b < n; ++b) {
    toff_q[b] = aq;
    toff_k[b] = ak;
    int lq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
    if (lq < 0 || lk < 0) bad = true;
    if (lq > max_seqlen || lk > max_seqlen) atomicOr(err, kErrSeqTooLong);
    aq += (max(lq, 0) + kTile - 1) / kTile;
    ak += (max(lk, 0) + kTile - 1) / kTile;
  }
  toff_q[n] = aq;
  toff_k[n] = ak;
  if (aq > cap_q || ak > cap_k) atomicOr(err, kErrTileOverflow);
  if (bad) atomicOr(err, kErrBadCuSeqlens);
}

// ---------------------------------------------------------------- K sums / V absmax
// grid (chunks of 512 tokens, H, nseq), 256 threads.  IS_K: exact channel
// sums of K (int64 fixed point for fp16, fp64 for bf16); else channel |max|
// of V (float bits, atomicMax on non-negative floats orders like uints).
template <int D, bool IS_K>
__global__ void __launch_bounds__(256) kv_stats_kernel(PrepassParams p) {
  constexpr int TPR = D / 8, RPI = 256 / TPR, CH = 512;
  __shared__ unsigned long long red[RPI][D];
  const int b = blockIdx.z, h = blockIdx.y;
  int start, len, toff;
  p.seqs.k(b, start, len, toff);                 // K and V share the key sequence ranges
  if (len > p.seqs.max_seqlen && p.seqs.cu_k) return;   // reported by the offsets kernel
  const int t0 = blockIdx.x * CH;
  if (t0 >= len) return;
  const int t1 = min(len, t0 + CH);
  const int cc = threadIdx.x % TPR, r0 = threadIdx.x / TPR;
  const uint16_t* base = p.x + (long long)b * p.st.sb + (long long)h * p.st.sh + cc * 8;
  long long ai[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  double ad[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float am[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int t = t0 + r0; t < t1; t += RPI) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (long long)(start + t) * p.st.ss));
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (IS_K) {
        if (p.bf16) ad[u] += (double)h16_to_f32(hv[u], true);
        else ai[u] += f16_fixed24(hv[u]);
      } else {
        am[u] = fmaxf(am[u], fabsf(h16_to_f32(hv[u], p.bf16)));
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    unsigned long long w;
    if (IS_K) w = p.bf16 ? (unsigned long long)__double_as_longlong(ad[u]) : (unsigned long long)ai[u];
    else w = __float_as_uint(am[u]);
    red[r0][cc * 8 + u] = w;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    const size_t o = ((size_t)b * p.H + h) * D + c;
    if (IS_K) {
      if (p.bf16) {
        double s = 0.0;
        for (int r = 0; r < RPI; ++r) s += __longlong_as_double((long long)red[r][c]);
        atomicAdd(reinterpret_cast<double*>(&p.k_stat[o]), s);
      } else {
        long long s = 0;
        for (int r = 0; r < RPI; ++r) s += (long long)red[r][c];
        atomicAdd(&p.k_stat[o], (unsigned long long)s);
      }
    } else {
      uint32_t m = 0;
      for (int r = 0; r < RPI; ++r) m = max(m, (uint32_t)red[r][c]);
      atomicMax(&p.v_stat[o], m);
    }
  }
}

// ---------------------------------------------------------------- Q / K INT8
// grid (tiles per sequence, H, nseq), 256 threads; one 128-token tile.
template <int D, bool IS_Q>
__global__ void __launch_bounds__(256) quant_qk_kernel(PrepassParams p) {
  constexpr int TPR = D / 8, RPI = 256 / TPR, NR = kTile / RPI;
  __shared__ float rowmax[kTile];
  __shared__ float gmax[kQGroupsMax];
  __shared__ float mu_s[D];
  __shared__ double dred[RPI][D];
  const int b = blockIdx.z, h = blockIdx.y, tile = blockIdx.x;
  int start, len, toff;
  if (IS_Q) p.seqs.q(b, start, len, toff); else p.seqs.k(b, start, len, toff);
  if ((p.seqs.cu_q || p.seqs.cu_k) && len > p.seqs.max_seqlen) return;
  if (tile * kTile >= len) return;
  const int tg = toff + tile;
  if (tg >= p.tiles) return;                             // reported by the offsets kernel
  const int tid = threadIdx.x, cc = tid % TPR, r0 = tid / TPR;
  const uint16_t* base = p.x + (long long)b * p.st.sb + (long long)h * p.st.sh + cc * 8;

  float x[NR][8];
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = r0 + RPI * i, t = tile * kTile + r;
    if (t < len) {
      uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (long long)(start + t) * p.st.ss));
      unpack8(v, p.bf16, x[i]);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) x[i][u] = 0.f;
    }
  }
  const int nvalid = min(kTile, len - tile * kTile);

  if (p.smooth) {
    if (IS_Q) {
      // block mean: exact fp64 sum of <= 128 16-bit values per channel
      double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int u = 0; u < 8; ++u) s[u] += (double)x[i][u];
#pragma unroll
      for (int u = 0; u < 8; ++u) dred[r0][cc * 8 + u] = s[u];
      __syncthreads();
      if (tid < D) {
        double a = 0.0;
        for (int r = 0; r < RPI; ++r) a += dred[r][tid];
        const float m = (float)(a / (double)nvalid);
        mu_s[tid] = m;
        p.q_mean[((size_t)h * p.tiles + tg) * D + tid] = m;
      }
    } else if (tid < D) {
      // channel mean over the whole sequence from the exact sums
      const unsigned long long w = p.k_stat[((size_t)b * p.H + h) * D + tid];
      const double sum = p.bf16 ? __longlong_as_double((long long)w) : (double)(long long)w * 0x1p-24;
      const float m = (float)(sum / (double)len);
      mu_s[tid] = m;
      if (tile == 0) p.k_mean[((size_t)b * p.H + h) * D + tid] = m;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int t = tile * kTile + r0 + RPI * i;
#pragma unroll
      for (int u = 0; u < 8; ++u) x[i][u] = (t < len) ? __fsub_rn(x[i][u], mu_s[cc * 8 + u]) : 0.f;
    }
  } else if (!IS_Q && tid < D && tile == 0) {
    p.k_mean[((size_t)b * p.H + h) * D + tid] = 0.f;
  }

  // row |max| (reduce the TPR lanes of a row), then group |max|
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) m = fmaxf(m, fabsf(x[i][u]));
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (cc == 0) rowmax[r0 + RPI * i] = m;
  }
  __syncthreads();
  const int ng = IS_Q ? q_ngroups(p.gran) : k_ngroups(p.gran);
  const int warp = tid >> 5, lane = tid & 31;
  for (int g = warp; g < ng; g += 8) {
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = lane + 32 * k;
      const int gr = IS_Q ? q_group(p.gran, r) : k_group(p.gran, r);
      if (gr == g && r < nvalid) m = fmaxf(m, rowmax[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      gmax[g] = m;
      p.scales[((size_t)h * p.tiles + tg) * (IS_Q ? kQGroupsMax : kKGroupsMax) + g] = __fdiv_rn(m, 127.0f);
    }
  }
  __syncthreads();

  int8_t* tbase = p.codes + ((size_t)h * p.tiles + tg) * (size_t)(kTile * D);
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = r0 + RPI * i;
    const float am = gmax[IS_Q ? q_group(p.gran, r) : k_group(p.gran, r)];
    const float inv = am > 0.f ? __fdiv_rn(127.0f, am) : 0.f;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      int c = __float2int_rn(__fmul_rn(x[i][u], inv));
      c = max(-127, min(127, c));
      w[u >> 2] |= ((uint32_t)(c & 0xFF)) << ((u & 3) * 8);
    }
    *reinterpret_cast<uint2*>(tbase + swz(r, cc * 8, D)) = make_uint2(w[0], w[1]);
  }
}

// ---------------------------------------------------------------- V
// grid (tiles per sequence, Hkv, nseq), 256 threads.  The 128 x D tile is
// staged in shared memory, then written transposed: FP8 rows of 128 keys, or
// 16-bit rows split in two 64-key halves.
template <int D, bool PV8>
__global__ void __launch_bounds__(256) quant_v_kernel(PrepassParams p) {
  constexpr int TPR = D / 8, RPI = 256 / TPR, NR = kTile / RPI;
  __shared__ __align__(16) uint16_t vt[kTile][D];
  __shared__ float inv_s[D];
  const int b = blockIdx.z, h = blockIdx.y, tile = blockIdx.x;
  int start, len, toff;
  p.seqs.k(b, start, len, toff);
  if (p.seqs.cu_k && len > p.seqs.max_seqlen) return;
  if (tile * kTile >= len) return;
  const int tg = toff + tile;
  if (tg >= p.tiles) return;
  const int tid = threadIdx.x, cc = tid % TPR, r0 = tid / TPR;
  const uint16_t* base = p.x + (long long)b * p.st.sb + (long long)h * p.st.sh + cc * 8;
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = r0 + RPI * i, t = tile * kTile + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < len) v = __ldg(reinterpret_cast<const uint4*>(base + (long long)(start + t) * p.st.ss));
    *reinterpret_cast<uint4*>(&vt[r][cc * 8]) = v;
  }
  if (PV8 && tid < D) {
    const float am = __uint_as_float(p.v_stat[((size_t)b * p.H + h) * D + tid]);
    inv_s[tid] = am > 0.f ? __fdiv_rn(kFp8Max, am) : 0.f;
    if (tile == 0) p.v_scale[((size_t)b * p.H + h) * D + tid] = __fdiv_rn(am, kFp8Max);
  }
  __syncthreads();
  uint8_t* tb = p.v_codes + ((size_t)h * p.tiles + tg) * (size_t)(D * kTile * (PV8 ? 1 : 2));
  if (PV8) {
    // output chunk (channel c, keys 16k..16k+15): 16 E4M3 codes
    for (int w = tid; w < D * 8; w += 256) {
      const int c = w % D, k = w / D;
      const float inv = inv_s[c];
      uint32_t o[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float f[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __fmul_rn(h16_to_f32(vt[16 * k + 4 * q4 + i][c], p.bf16), inv);
        o[q4] = pack_e4m3x4(f[0], f[1], f[2], f[3]);
      }
      *reinterpret_cast<uint4*>(tb + swz(c, 16 * k, 128)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    // output chunk (half hf, channel c, keys 64hf + 8kk .. +7): 8 16-bit values
    for (int w = tid; w < D * 16; w += 256) {
      const int c = w % D, k = w / D, hf = k >> 3, kk = k & 7;
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = 64 * hf + 8 * kk + 2 * i;
        o[i] = (uint32_t)vt[key][c] | ((uint32_t)vt[key + 1][c] << 16);
      }
      *reinterpret_cast<uint4*>(tb + (size_t)hf * (D * 128) + swz(c, 16 * kk, 128)) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ---------------------------------------------------------------- launchers
template <int D>
static cudaError_t launch_qk(const PrepassParams& pq, const PrepassParams& pk, int nseq, int tps_q,
                             int tps_k, cudaStream_t s) {
  kv_stats_kernel<D, true><<<dim3((pk.seqs.max_seqlen + 511) / 512, pk.H, nseq), 256, 0, s>>>(pk);
  quant_qk_kernel<D, true><<<dim3(tps_q, pq.H, nseq), 256, 0, s>>>(pq);
  quant_qk_kernel<D, false><<<dim3(tps_k, pk.H, nseq), 256, 0, s>>>(pk);
  return cudaGetLastError();
}

cudaError_t prepass_qk(const PrepassParams& pq, const PrepassParams& pk, int D, int nseq, int tps_q,
                       int tps_k, cudaStream_t s) {
  return D == 128 ? launch_qk<128>(pq, pk, nseq, tps_q, tps_k, s)
                  : launch_qk<64>(pq, pk, nseq, tps_q, tps_k, s);
}

template <int D, bool PV8>
static cudaError_t launch_v(const PrepassParams& pv, int nseq, int tps, cudaStream_t s) {
  if (PV8)
    kv_stats_kernel<D, false><<<dim3((pv.seqs.max_seqlen + 511) / 512, pv.H, nseq), 256, 0, s>>>(pv);
  quant_v_kernel<D, PV8><<<dim3(tps, pv.H, nseq), 256, 0, s>>>(pv);
  return cudaGetLastError();
}

cudaError_t prepass_v(const PrepassParams& pv, int D, bool pv8, int nseq, int tps, cudaStream_t s) {
  if (D == 128) return pv8 ? launch_v<128, true>(pv, nseq, tps, s) : launch_v<128, false>(pv, nseq, tps, s);
  return pv8 ? launch_v<64, true>(pv, nseq, tps, s) : launch_v<64, false>(pv, nseq, tps, s);
}

cudaError_t prepass_varlen_offsets(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q,
                                   int cap_k, int* toff_q, int* toff_k, uint32_t* err, cudaStream_t s) {
  varlen_offsets_kernel<<<1, 32, 0, s>>>(cu_q, cu_k, n, max_seqlen, cap_q, cap_k, toff_q, toff_k, err);
  return cudaGetLastError();
}

}  // namespace sage
