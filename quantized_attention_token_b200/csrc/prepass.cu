// prepass.cu -- smooth + quantize pre-pass (HBM-bound): two streaming launches.
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
// Launches.  The K mean and the V maxima need every token of a sequence
// before any K / V tile can be quantized, so the pre-pass is two grids of
// short-lived CTAs, each CTA one 128-token tile of one head:
//   A: Q tiles -> INT8 codes and group scales (smoothed by the block mean when
//      Q smoothing is on); K tiles -> exact channel sums; V tiles -> channel
//      |max| (FP8 mode), both added atomically into per-(sequence, KV head)
//      accumulators that are zeroed before the launch.
//   B: K tiles -> INT8 codes of K - mean; V tiles -> E4M3 codes (or the 16-bit
//      values) written transposed.  B visits the K / V tiles in the reverse of
//      A's order, so the tiles A read last, still in L2, are the first B reads.
// Each thread loads its whole share of a tile (eight or four 16-byte loads)
// before any arithmetic, and several CTAs share an SM, so one CTA's barrier
// waits overlap the others' loads.
//
// A one-pass alternative for K and V (debug-selected, see
// prepass_kv_cluster_kernel) reads them from HBM once: one thread-block
// cluster per (tensor, sequence, KV head) holds the head in shared memory.
// It writes the same bytes; on B200 it measured slower than the two launches.
#include "sage_launch.cuh"

namespace sage {

constexpr int kPrepassThreads = 256;
// Resident CTAs per SM the pre-pass launches are built for.  D = 64 threads
// hold half as many 16-byte chunks of a tile (4), so a fourth CTA keeps more
// loads in flight: 0.196 vs 0.224 ms at B=8 H=32 S=4096 D=64 on B200, without
// spills.  At D = 128 a fourth CTA left 64 registers and made the kernels spill
// (108-228 bytes), for no gain at B=2 H=32 S=4096.
template <int D>
constexpr int prepass_min_ctas() { return D == 64 ? 4 : 3; }

// Thread (cc = tid % TPR, rg = tid / TPR) owns 16-byte chunk cc (channels
// 8cc .. 8cc+7) of the NR consecutive rows rg*NR .. rg*NR + NR-1.
template <int D>
struct Map {
  static constexpr int TPR = D / 8;
  static constexpr int RG = kPrepassThreads / TPR;
  static constexpr int NR = kTile / RG;
  static constexpr int WARPS = kPrepassThreads / 32;
};

// Read-only 16-byte loads.  ld_keep leaves the line to L2's normal policy (K
// and V in launch A are read again by launch B); ld_last marks it for early
// eviction (its last use).
__device__ __forceinline__ uint4 ld_keep(const uint16_t* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ld_last(const uint16_t* p, uint64_t pol) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint16_t h16(const uint4& v, int u) { return reinterpret_cast<const uint16_t*>(&v)[u]; }

// ---------------------------------------------------------------- tile -> sequence
struct TileLoc {
  int b, tile, start, len, nvalid;
};

// Workspace tile slot t of a head -> its sequence and the tile's token range.
// False when t holds no tokens (past the last tile, or a varlen sequence whose
// bad length the offsets kernel has flagged).
__device__ __forceinline__ bool locate(const PrepassJob& j, bool is_q, int t, TileLoc& L) {
  const Seqs& s = j.seqs;
  if (!s.cu_k) {
    L.b = t / s.tps;
    L.tile = t - L.b * s.tps;
    if (L.b >= j.nseq) return false;
    L.start = 0;
    L.len = s.S;
  } else {
    const int* toff = is_q ? s.toff_q : s.toff_k;
    if (t >= toff[j.nseq]) return false;
    int lo = 0, hi = j.nseq - 1;             // the last b with toff[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (toff[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int* cu = is_q ? s.cu_q : s.cu_k;
    L.b = lo;
    L.tile = t - toff[lo];
    L.start = cu[lo];
    L.len = cu[lo + 1] - cu[lo];
    if (L.len < 0 || L.len > s.max_seqlen) return false;
  }
  L.nvalid = min(kTile, L.len - L.tile * kTile);
  return L.nvalid > 0;
}

// The thread's NR chunks of the tile (zeros past the sequence).
template <int D, bool LAST>
__device__ __forceinline__ void load_tile(const uint16_t* head, long long ss, const TileLoc& L,
                                          uint4 (&v)[Map<D>::NR]) {
  using M = Map<D>;
  const int cc = threadIdx.x % M::TPR, rg = threadIdx.x / M::TPR;
  const uint16_t* p = head + (long long)(L.start + L.tile * kTile + rg * M::NR) * ss + cc * 8;
  uint64_t pol = 0;
  if (LAST) pol = policy_evict_first();
#pragma unroll
  for (int i = 0; i < M::NR; ++i) {
    if (rg * M::NR + i < L.nvalid) v[i] = LAST ? ld_last(p + i * ss, pol) : ld_keep(p + i * ss);
    else v[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// ---------------------------------------------------------------- shared memory
template <int D>
struct QuantSmem {
  double red[Map<D>::WARPS][D];   // block-mean partial sums (smooth Q)
  float mu[D];
  float rowmax[kTile];
  float ginv[kQGroupsMax];        // 127 / group amax (0 for an all-zero group)
};
template <int D>
struct StatSmem {
  double sum[Map<D>::WARPS][D];
  uint32_t amax[Map<D>::WARPS][D];
  uint32_t kneg[Map<D>::WARPS][D];   // smooth V: keys of the negated values
};

// Order-preserving 16-bit key of a finite fp16 / bf16 bit pattern (larger
// value, larger key) and its inverse.
__device__ __forceinline__ uint32_t key16(uint16_t h) {
  return (h & 0x8000u) ? (~(uint32_t)h & 0xFFFFu) : ((uint32_t)h | 0x8000u);
}
__device__ __forceinline__ uint16_t unkey16(uint32_t k) {
  return (k & 0x8000u) ? (uint16_t)(k ^ 0x8000u) : (uint16_t)(~k & 0xFFFFu);
}
template <int D>
struct VSmem {
  float inv[D];                   // 448 / channel amax (FP8 mode)
  float mu[D];                    // channel mean (smooth V), else 0
};
template <int D>
struct VTileSmem {
  VSmem<D> v;
  uint32_t tile[kTile * D / 2];   // the 16-bit tile, row-major, two values per word
};

// Sum or max of a per-lane value over the lanes of a warp that own the same
// channel chunk (lanes l, l ^ TPR, ...).
template <int D, class T, class Op>
__device__ __forceinline__ T reduce_same_chunk(T x, Op op) {
#pragma unroll
  for (int o = Map<D>::TPR; o < 32; o <<= 1) x = op(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// ---------------------------------------------------------------- Q / K tile
// INT8 codes and group scales of one Q tile (launch A) or K tile (launch B);
// for K also the channel mean (written once per sequence and head).
// v: the thread's NR chunks of the tile (zeros past the sequence).
template <int D, bool IS_Q, bool BF16>
__device__ void quant_tile(const PrepassJob& j, int h, int t, const TileLoc& L, QuantSmem<D>& sm,
                           const uint4 (&v)[Map<D>::NR]) {
  using M = Map<D>;
  const int tid = threadIdx.x, cc = tid % M::TPR, rg = tid / M::TPR, warp = tid >> 5, lane = tid & 31;
  const int H = IS_Q ? j.Hq : j.Hkv;
  const int tiles = IS_Q ? j.tiles_q : j.tiles_k;

  const bool smooth = IS_Q ? j.smooth_q : j.smooth_k;
  if (smooth) {
    if (IS_Q) {
      // block mean: exact fp64 sums of <= 128 16-bit values per channel
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        double a = 0.0;
#pragma unroll
        for (int i = 0; i < M::NR; ++i) a += (double)h16_to_f32(h16(v[i], u), BF16);
        a = reduce_same_chunk<D>(a, [](double x, double y) { return x + y; });
        if (lane < M::TPR) sm.red[warp][cc * 8 + u] = a;
      }
      __syncthreads();
      if (tid < D) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < M::WARPS; ++w) s += sm.red[w][tid];
        const float m = (float)(s / (double)L.nvalid);
        sm.mu[tid] = m;
        j.q_mean[((size_t)h * tiles + t) * D + tid] = m;
      }
    } else if (tid < D) {
      // channel mean over the whole sequence from the exact sums
      const unsigned long long w = __ldcg(&j.k_stat[((size_t)L.b * H + h) * D + tid]);
      const double sum = BF16 ? __longlong_as_double((long long)w) : (double)(long long)w * 0x1p-24;
      const float m = (float)(sum / (double)L.len);
      sm.mu[tid] = m;
      if (L.tile == 0) j.k_mean[((size_t)L.b * H + h) * D + tid] = m;
    }
    __syncthreads();
  } else if (!IS_Q && tid < D && L.tile == 0) {
    j.k_mean[((size_t)L.b * H + h) * D + tid] = 0.f;
  }
  float mu[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) mu[u] = smooth ? sm.mu[cc * 8 + u] : 0.f;
  // the smoothed values of row i's chunk (0 past the sequence)
  auto X8 = [&](int i, float (&x)[8]) {
    const bool valid = rg * M::NR + i < L.nvalid;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float f = h16_to_f32(h16(v[i], u), BF16);
      x[u] = valid ? (smooth ? __fsub_rn(f, mu[u]) : f) : 0.f;
    }
  };
  // row |max| (over the TPR lanes of a row)
#pragma unroll
  for (int i = 0; i < M::NR; ++i) {
    float x[8];
    X8(i, x);
    float m = max3(fabsf(x[0]), fabsf(x[1]), fabsf(x[2]));
    m = max3(m, fabsf(x[3]), fabsf(x[4]));
    m = max3(m, fabsf(x[5]), fabsf(x[6]));
    m = fmaxf(m, fabsf(x[7]));
#pragma unroll
    for (int o = M::TPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (cc == 0) {
      const int r = rg * M::NR + i;
      if (IS_Q && j.gran == 3) {
        // per-token Q: the row is its own group (rows past the sequence: 0)
        const float am = r < L.nvalid ? m : 0.f;
        sm.ginv[r] = am > 0.f ? __fdiv_rn(127.0f, am) : 0.f;
        j.q_scale[((size_t)h * tiles + t) * kQGroupsMax + r] = __fdiv_rn(am, 127.0f);
      } else {
        sm.rowmax[r] = m;
      }
    }
  }
  __syncthreads();
  // group |max| -> the scale amax / 127 and the multiplier 127 / amax
  const int ng = (IS_Q && j.gran == 3) ? 0 : IS_Q ? q_ngroups(j.gran) : k_ngroups(j.gran);
  for (int g = warp; g < ng; g += M::WARPS) {
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < kTile / 32; ++k) {
      const int r = lane + 32 * k;
      const int gr = IS_Q ? q_group(j.gran, r) : k_group(j.gran, r);
      if (gr == g && r < L.nvalid) m = fmaxf(m, sm.rowmax[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      sm.ginv[g] = m > 0.f ? __fdiv_rn(127.0f, m) : 0.f;
      float* s = IS_Q ? j.q_scale : j.k_scale;
      s[((size_t)h * tiles + t) * (IS_Q ? kQGroupsMax : kKGroupsMax) + g] = __fdiv_rn(m, 127.0f);
    }
  }
  __syncthreads();
  int8_t* tbase = (IS_Q ? j.q_codes : j.k_codes) + ((size_t)h * tiles + t) * (size_t)(kTile * D);
#pragma unroll
  for (int i = 0; i < M::NR; ++i) {
    const int r = rg * M::NR + i;
    const float inv = sm.ginv[IS_Q ? q_group(j.gran, r) : k_group(j.gran, r)];
    float x[8];
    X8(i, x);
    // code = rne(x * inv): adding 1.5 * 2^23 rounds the product to an integer
    // (ties to even) and leaves it, two's complement, in the low bits.  No
    // clamp is needed: |x| <= amax and inv = fl(127/amax) give |x * inv| <=
    // 127 (1 + 2^-24), which rounds to at most 127.
    uint32_t b[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) b[u] = __float_as_uint(__fadd_rn(__fmul_rn(x[u], inv), 12582912.0f));
    const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    *reinterpret_cast<uint2*>(tbase + swz(r, cc * 8, D)) = make_uint2(w0, w1);
  }
}

// ---------------------------------------------------------------- K / V statistics
// Channel sums of a K tile, exact: for fp16 every partial sum of <= 128 values
// is a multiple of 2^-24 below 2^23 in magnitude, so fp64 holds it exactly and
// it is added as a 2^-24 fixed-point int64 (bf16: added as fp64).
template <int D, bool BF16>
__device__ void kstat_tile(const PrepassJob& j, int h, const TileLoc& L, StatSmem<D>& sm,
                           const uint4 (&v)[Map<D>::NR]) {
  using M = Map<D>;
  const int tid = threadIdx.x, cc = tid % M::TPR, warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    double a = 0.0;
#pragma unroll
    for (int i = 0; i < M::NR; ++i) a += (double)h16_to_f32(h16(v[i], u), BF16);
    a = reduce_same_chunk<D>(a, [](double x, double y) { return x + y; });
    if (lane < M::TPR) sm.sum[warp][cc * 8 + u] = a;
  }
  __syncthreads();
  if (tid < D) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < M::WARPS; ++w) s += sm.sum[w][tid];
    unsigned long long* dst = &j.k_stat[((size_t)L.b * j.Hkv + h) * D + tid];
    if (BF16) atomicAdd(reinterpret_cast<double*>(dst), s);
    else atomicAdd(dst, (unsigned long long)(long long)(s * 0x1p24));
  }
}

// Channel |max| of a V tile (|x| bit patterns of 16-bit floats order like the
// values).  Smooth V: the exact channel sums (as for K) and the keys of the
// channel maximum and of the negated minimum, from which launch B gets the
// mean and |max| of V - mean: float32 subtraction of a fixed mean is monotone,
// so that |max| comes from the two extremes.
template <int D, bool BF16, bool SMOOTH>
__device__ void vstat_tile(const PrepassJob& j, int h, const TileLoc& L, StatSmem<D>& sm,
                           const uint4 (&v)[Map<D>::NR]) {
  using M = Map<D>;
  const int tid = threadIdx.x, cc = tid % M::TPR, rg = tid / M::TPR, warp = tid >> 5, lane = tid & 31;
  const size_t o = ((size_t)L.b * j.Hkv + h) * D;
  if constexpr (!SMOOTH) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      uint32_t a = 0;
#pragma unroll
      for (int i = 0; i < M::NR; ++i) a = max(a, (uint32_t)(h16(v[i], u) & 0x7FFF));
      a = reduce_same_chunk<D>(a, [](uint32_t x, uint32_t y) { return max(x, y); });
      if (lane < M::TPR) sm.amax[warp][cc * 8 + u] = a;
    }
    __syncthreads();
    if (tid < D) {
      uint32_t m = 0;
#pragma unroll
      for (int w = 0; w < M::WARPS; ++w) m = max(m, sm.amax[w][tid]);
      atomicMax(&j.v_stat[2 * (o + tid)], __float_as_uint(h16_to_f32((uint16_t)m, BF16)));
    }
    return;
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      double a = 0.0;
      uint32_t kmax = 0, kneg = 0;
#pragma unroll
      for (int i = 0; i < M::NR; ++i) {
        const uint16_t x = h16(v[i], u);
        a += (double)h16_to_f32(x, BF16);                 // rows past the sequence hold 0
        if (rg * M::NR + i < L.nvalid) {
          kmax = max(kmax, key16(x));
          kneg = max(kneg, key16(x ^ 0x8000u));
        }
      }
      a = reduce_same_chunk<D>(a, [](double x, double y) { return x + y; });
      kmax = reduce_same_chunk<D>(kmax, [](uint32_t x, uint32_t y) { return max(x, y); });
      kneg = reduce_same_chunk<D>(kneg, [](uint32_t x, uint32_t y) { return max(x, y); });
      if (lane < M::TPR) {
        sm.sum[warp][cc * 8 + u] = a;
        sm.amax[warp][cc * 8 + u] = kmax;
        sm.kneg[warp][cc * 8 + u] = kneg;
      }
    }
    __syncthreads();
    if (tid < D) {
      double sum = 0.0;
      uint32_t kmax = 0, kneg = 0;
#pragma unroll
      for (int w = 0; w < M::WARPS; ++w) {
        sum += sm.sum[w][tid];
        kmax = max(kmax, sm.amax[w][tid]);
        kneg = max(kneg, sm.kneg[w][tid]);
      }
      if (BF16) atomicAdd(reinterpret_cast<double*>(&j.v_sum[o + tid]), sum);
      else atomicAdd(&j.v_sum[o + tid], (unsigned long long)(long long)(sum * 0x1p24));
      atomicMax(&j.v_stat[2 * (o + tid)], kmax);
      atomicMax(&j.v_stat[2 * (o + tid) + 1], kneg);
    }
  }
}

// ---------------------------------------------------------------- V tile
// V written transposed: FP8 rows of 128 keys, or 16-bit rows split in two
// 64-key halves.  `tile` is the 16-bit tile in shared memory, row-major, two
// values per 32-bit word, rows past the sequence zero; the caller makes it
// visible to the whole CTA before the first barrier below.  Each output unit
// gathers two adjacent channels (one 32-bit word per key).
template <int D, bool BF16, bool SMOOTH>
__device__ void v_tile(const PrepassJob& j, int h, int t, const TileLoc& L, VSmem<D>& sm, const uint32_t* tile) {
  const int tid = threadIdx.x;
  if (j.pv8 && tid < D) {
    const size_t o = ((size_t)L.b * j.Hkv + h) * D + tid;
    float am, mu = 0.f;
    if (SMOOTH) {
      // the channel mean from the exact sum, then |max| of V - mean
      const unsigned long long w = __ldcg(&j.v_sum[o]);
      const double sum = BF16 ? __longlong_as_double((long long)w) : (double)(long long)w * 0x1p-24;
      mu = (float)(sum / (double)L.len);
      const float vmax = h16_to_f32(unkey16(__ldcg(&j.v_stat[2 * o])), BF16);
      const float vmin = -h16_to_f32(unkey16(__ldcg(&j.v_stat[2 * o + 1])), BF16);
      am = fmaxf(fabsf(__fsub_rn(vmax, mu)), fabsf(__fsub_rn(vmin, mu)));
      if (L.tile == 0) j.v_mean[o] = mu;
    } else {
      am = __uint_as_float(__ldcg(&j.v_stat[2 * o]));
    }
    sm.mu[tid] = mu;
    sm.inv[tid] = am > 0.f ? __fdiv_rn(kFp8Max, am) : 0.f;
    if (L.tile == 0) j.v_scale[o] = __fdiv_rn(am, kFp8Max);
  }
  __syncthreads();
  uint8_t* tb = j.v_codes + ((size_t)h * j.tiles_k + t) * (size_t)(D * kTile * (j.pv8 ? 1 : 2));
  if (j.pv8) {
    // unit (channel pair p, keys 16k .. 16k+15): two 16-byte runs of E4M3 codes
    for (int w = tid; w < (D / 2) * 8; w += kPrepassThreads) {
      const int p = w % (D / 2), k = w / (D / 2);
      const float i0 = sm.inv[2 * p], i1 = sm.inv[2 * p + 1];
      const float m0 = SMOOTH ? sm.mu[2 * p] : 0.f, m1 = SMOOTH ? sm.mu[2 * p + 1] : 0.f;
      uint32_t o0[4], o1[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float f0[4], f1[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = 16 * k + 4 * q4 + e;
          const uint32_t x = tile[key * (D / 2) + p];
          const float x0 = h16_to_f32((uint16_t)(x & 0xFFFF), BF16), x1 = h16_to_f32((uint16_t)(x >> 16), BF16);
          if (SMOOTH) {        // (V - mean) * 448 / |max|; keys past the sequence stay 0
            const bool in = key < L.nvalid;
            f0[e] = in ? __fmul_rn(__fsub_rn(x0, m0), i0) : 0.f;
            f1[e] = in ? __fmul_rn(__fsub_rn(x1, m1), i1) : 0.f;
          } else {             // rows past the sequence hold 0
            f0[e] = __fmul_rn(x0, i0);
            f1[e] = __fmul_rn(x1, i1);
          }
        }
        o0[q4] = pack_e4m3x4(f0[0], f0[1], f0[2], f0[3]);
        o1[q4] = pack_e4m3x4(f1[0], f1[1], f1[2], f1[3]);
      }
      *reinterpret_cast<uint4*>(tb + swz(2 * p, 16 * k, 128)) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
      *reinterpret_cast<uint4*>(tb + swz(2 * p + 1, 16 * k, 128)) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
    }
  } else {
    // unit (channel pair p, keys 8o .. 8o+7): two 16-byte runs of 16-bit values
    for (int w = tid; w < (D / 2) * 16; w += kPrepassThreads) {
      const int p = w % (D / 2), o = w / (D / 2), hf = o >> 3, kk = o & 7;
      uint32_t x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = tile[(8 * o + e) * (D / 2) + p];
      uint32_t a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = __byte_perm(x[2 * i], x[2 * i + 1], 0x5410);   // channel 2p: keys 2i, 2i+1
        b[i] = __byte_perm(x[2 * i], x[2 * i + 1], 0x7632);   // channel 2p+1
      }
      uint8_t* half = tb + (size_t)hf * (D * 128);
      *reinterpret_cast<uint4*>(half + swz(2 * p, 16 * kk, 128)) = make_uint4(a[0], a[1], a[2], a[3]);
      *reinterpret_cast<uint4*>(half + swz(2 * p + 1, 16 * kk, 128)) = make_uint4(b[0], b[1], b[2], b[3]);
    }
  }
}

// ---------------------------------------------------------------- kernels
// Launch A: blockIdx.x = tile slot, blockIdx.y over [Q heads | K-statistics
// heads | V-statistics heads] (each part present only when asked for).
template <int D, bool BF16, bool SV>
__global__ void __launch_bounds__(kPrepassThreads, prepass_min_ctas<D>()) prepass_a_kernel(const PrepassJob j) {
  __shared__ union {
    QuantSmem<D> q;
    StatSmem<D> s;
  } sm;
  const int t = blockIdx.x;
  int y = blockIdx.y;
  const int nq = j.do_q ? j.Hq : 0;
  const int nks = (j.do_k && j.smooth_k) ? j.Hkv : 0;
  TileLoc L;
  uint4 v[Map<D>::NR];
  if (y < nq) {
    if (t < j.tiles_q && locate(j, true, t, L)) {
      load_tile<D, true>(j.q + (long long)L.b * j.sq.sb + (long long)y * j.sq.sh, j.sq.ss, L, v);
      quant_tile<D, true, BF16>(j, y, t, L, sm.q, v);
    }
  } else if ((y -= nq) < nks) {
    if (t < j.tiles_k && locate(j, false, t, L)) {
      load_tile<D, false>(j.k + (long long)L.b * j.sk.sb + (long long)y * j.sk.sh, j.sk.ss, L, v);
      kstat_tile<D, BF16>(j, y, L, sm.s, v);
    }
  } else {
    y -= nks;
    if (t < j.tiles_k && locate(j, false, t, L)) {
      load_tile<D, false>(j.v + (long long)L.b * j.sv.sb + (long long)y * j.sv.sh, j.sv.ss, L, v);
      vstat_tile<D, BF16, SV>(j, y, L, sm.s, v);
    }
  }
}

// Launch B: blockIdx.y over [K heads | V heads], both axes walked backwards
// (the last V head's last tile first).
template <int D, bool BF16, bool SV>
__global__ void __launch_bounds__(kPrepassThreads, prepass_min_ctas<D>()) prepass_b_kernel(const PrepassJob j) {
  __shared__ union {
    QuantSmem<D> q;
    VTileSmem<D> vt;
  } sm;
  const int t = gridDim.x - 1 - blockIdx.x;
  const int y = gridDim.y - 1 - blockIdx.y;
  const int nk = j.do_k ? j.Hkv : 0;
  TileLoc L;
  if (!locate(j, false, t, L)) return;
  uint4 v[Map<D>::NR];
  if (y < nk) {
    load_tile<D, true>(j.k + (long long)L.b * j.sk.sb + (long long)y * j.sk.sh, j.sk.ss, L, v);
    quant_tile<D, false, BF16>(j, y, t, L, sm.q, v);
  } else {
    const int h = y - nk;
    load_tile<D, true>(j.v + (long long)L.b * j.sv.sb + (long long)h * j.sv.sh, j.sv.ss, L, v);
    using M = Map<D>;
    const int cc = threadIdx.x % M::TPR, rg = threadIdx.x / M::TPR;
#pragma unroll
    for (int i = 0; i < M::NR; ++i)
      *reinterpret_cast<uint4*>(&sm.vt.tile[(rg * M::NR + i) * (D / 2) + cc * 4]) = v[i];
    v_tile<D, BF16, SV>(j, h, t, L, sm.vt.v, sm.vt.tile);
  }
}

// ---------------------------------------------------------------- K / V in one pass
// When every sequence's K (or V) of one head fits in the shared memory of a
// thread-block cluster, one cluster per (tensor, sequence, KV head) reads it
// from HBM once: CTA `rank` copies tiles rank*TMAX .. rank*TMAX + TMAX-1 into
// its own shared memory, adds their statistics into the per-(sequence, head)
// accumulators (as launch A does), waits at the cluster barrier for the other
// CTAs' contributions, and then quantizes its tiles from shared memory (as
// launch B does).  The statistics meet in global memory: the accumulators are
// exact integer / max reductions, so their order does not matter, and the
// cluster barrier's release / acquire makes every CTA's atomics visible to
// the others.  No CTA reads another's shared memory.

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16-byte asynchronous global -> shared copy (plain form: whole source, no
// cache hint) and its group bookkeeping.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Wait until at most n (0..7) of this thread's groups are pending.
__device__ __forceinline__ void cp_async_wait_upto(int n) {
  switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
  }
}

// Start copying the thread's NR chunks of a tile into shared memory (rows of
// D 16-bit values, the layout load_staged and v_tile read); chunks past the
// sequence are zeroed with plain stores.
template <int D>
__device__ __forceinline__ void stage_tile(const uint16_t* head, long long ss, const TileLoc& L, uint32_t stage,
                                           uint8_t* stage_ptr) {
  using M = Map<D>;
  const int cc = threadIdx.x % M::TPR, rg = threadIdx.x / M::TPR;
  const uint16_t* p = head + (long long)(L.start + L.tile * kTile + rg * M::NR) * ss + cc * 8;
#pragma unroll
  for (int i = 0; i < M::NR; ++i) {
    const uint32_t off = (uint32_t)((rg * M::NR + i) * (D * 2) + cc * 16);
    if (rg * M::NR + i < L.nvalid) cp_async16(stage + off, p + i * ss);
    else *reinterpret_cast<uint4*>(stage_ptr + off) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// The thread's NR chunks of a tile staged in shared memory.
template <int D>
__device__ __forceinline__ void load_staged(const uint8_t* stage, uint4 (&v)[Map<D>::NR]) {
  using M = Map<D>;
  const int cc = threadIdx.x % M::TPR, rg = threadIdx.x / M::TPR;
#pragma unroll
  for (int i = 0; i < M::NR; ++i)
    v[i] = *reinterpret_cast<const uint4*>(stage + (size_t)(rg * M::NR + i) * (D * 2) + cc * 16);
}

// Tile ti of sequence b's keys: its token range and workspace slot t.  False
// when it holds no tokens, when the sequence's length is invalid (flagged by
// the offsets kernel) or when its slot lies past the workspace's tiles.
__device__ __forceinline__ bool locate_kv(const PrepassJob& j, int b, int ti, int& t, TileLoc& L) {
  const Seqs& s = j.seqs;
  L.b = b;
  L.tile = ti;
  if (!s.cu_k) {
    L.start = 0;
    L.len = s.S;
    t = b * s.tps + ti;
  } else {
    L.start = s.cu_k[b];
    L.len = s.cu_k[b + 1] - L.start;
    if (L.len < 0 || L.len > s.max_seqlen) return false;
    t = s.toff_k[b] + ti;
  }
  L.nvalid = min(kTile, L.len - ti * kTile);
  return L.nvalid > 0 && t < j.tiles_k;
}

template <int D>
__host__ __device__ constexpr int kv_tile_bytes() { return kTile * D * 2; }

// Cluster c (clusterid.x) is job c: jobs [0, n_k_jobs) are the K heads
// (sequence-major), the rest the V heads.  Dynamic shared memory: TMAX tiles.
template <int D, bool BF16, bool SV, int TMAX>
__global__ void __launch_bounds__(kPrepassThreads, 2) prepass_kv_cluster_kernel(const PrepassJob j, int n_k_jobs) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ union {
    QuantSmem<D> q;
    StatSmem<D> s;
    VSmem<D> v;
  } sm;
  constexpr int SB = kv_tile_bytes<D>();
  const int rank = (int)cluster_rank(), job = (int)cluster_index();
  const bool is_k = job < n_k_jobs;
  const int jb = is_k ? job : job - n_k_jobs;
  const int b = jb / j.Hkv, h = jb - b * j.Hkv;
  const Strides& st = is_k ? j.sk : j.sv;
  const uint16_t* head = (is_k ? j.k : j.v) + (long long)b * st.sb + (long long)h * st.sh;
  const uint32_t stage0 = (uint32_t)__cvta_generic_to_shared(stage_mem);
  // 1. all of this CTA's copies in flight, one group per tile
#pragma unroll
  for (int i = 0; i < TMAX; ++i) {
    TileLoc L;
    int t;
    if (locate_kv(j, b, rank * TMAX + i, t, L)) stage_tile<D>(head, st.ss, L, stage0 + i * SB, stage_mem + i * SB);
    cp_async_commit();
  }
  // 2. statistics of each tile as its copy lands: smooth K needs the channel
  //    sums, FP8 V the channel |max| (and, smooth V, sums and extremes)
  const bool stats = is_k ? (j.smooth_k != 0) : (j.pv8 != 0);
#pragma unroll
  for (int i = 0; i < TMAX; ++i) {
    cp_async_wait_upto(TMAX - 1 - i);
    TileLoc L;
    int t;
    if (stats && locate_kv(j, b, rank * TMAX + i, t, L)) {
      uint4 v[Map<D>::NR];
      load_staged<D>(stage_mem + i * SB, v);
      if (is_k) kstat_tile<D, BF16>(j, h, L, sm.s, v);
      else vstat_tile<D, BF16, SV>(j, h, L, sm.s, v);
      __syncthreads();             // sm.s is reused by the next tile
    }
  }
  cp_async_wait<0>();
  __syncthreads();                 // every staged tile visible to the whole CTA
  // 3. every CTA of the cluster has added its contributions
  cluster_sync_all();
  // 4. quantize from shared memory
#pragma unroll 1
  for (int i = 0; i < TMAX; ++i) {
    TileLoc L;
    int t;
    if (!locate_kv(j, b, rank * TMAX + i, t, L)) continue;
    if (is_k) {
      uint4 v[Map<D>::NR];
      load_staged<D>(stage_mem + i * SB, v);
      quant_tile<D, false, BF16>(j, h, t, L, sm.q, v);
    } else {
      v_tile<D, BF16, SV>(j, h, t, L, sm.v, reinterpret_cast<const uint32_t*>(stage_mem + i * SB));
    }
    __syncthreads();               // sm is reused by the next tile
  }
}

// ---------------------------------------------------------------- smooth-Q bias
// Launch C (smooth Q, dense problems): the score correction of every key for
// every query tile.  Q was smoothed by its block mean mu (per 128-row tile),
// so the scores lose mu . k_j; with k_j the dequantized smoothed key
// (delta_K[g(j)] * K_codes[j]) the correction of key j is
//   bias[h][tq][j] = (sum_c mu[tq][c] * K_codes[j][c]) * delta_K[g(j)],
// the same for every row of the tile.  The sum runs over c in order in fp64
// (float x int8 products are exact there) and is rounded to float once.
// One CTA of 128 threads (one per key) per (query tile, key tile, head).
template <int D>
__global__ void __launch_bounds__(kTile) qbias_kernel(const PrepassJob j, float* __restrict__ q_bias) {
  __shared__ double mu[D];
  const int tq = blockIdx.x, tk = blockIdx.y, h = blockIdx.z, r = threadIdx.x;
  const int tps = j.seqs.tps;
  const int b = tq / tps;
  if (b >= j.nseq) return;
  const int hk = h / j.group;
  const int ks = b * tps + tk;                      // the key tile's workspace slot
  if (r < D) mu[r] = (double)j.q_mean[((size_t)h * j.tiles_q + tq) * D + r];
  __syncthreads();
  const int8_t* row = j.k_codes + ((size_t)hk * j.tiles_k + ks) * (size_t)(kTile * D) + (size_t)r * D;
  double acc = 0.0;
#pragma unroll
  for (int cc = 0; cc < D / 16; ++cc) {
    const int4 w = *reinterpret_cast<const int4*>(row + (swz(r, cc * 16, D) - r * D));
    const int8_t* e = reinterpret_cast<const int8_t*>(&w);
#pragma unroll
    for (int u = 0; u < 16; ++u) acc += mu[cc * 16 + u] * (double)e[u];
  }
  const float dk = j.k_scale[((size_t)hk * j.tiles_k + ks) * kKGroupsMax + k_group(j.gran, r)];
  q_bias[((size_t)h * j.tiles_q + tq) * (size_t)(tps * kTile) + tk * kTile + r] = (float)(acc * (double)dk);
}

// ---------------------------------------------------------------- varlen offsets
// toff[b] = sum_{b'<b} ceil(L_b'/128) for q and k.  Checks the lengths against
// max_seqlen and the workspace's tile capacity.
__global__ void varlen_offsets_kernel(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q,
                                      int cap_k, int* toff_q, int* toff_k, uint32_t* err) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int aq = 0, ak = 0;
  bool bad = cu_q[0] != 0 || cu_k[0] != 0;
  for (int b = 0; b < n; ++b) {
    toff_q[b] = aq;
    toff_k[b] = ak;
    const int lq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
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

// ---------------------------------------------------------------- launchers
// Largest cluster the one-pass K / V path uses (16 needs the non-portable
// cluster-size opt-in) and the largest staged share of a CTA.
constexpr int kKvMaxCluster = 16;
template <int D>
constexpr int kv_max_tiles_per_cta() { return D == 128 ? 4 : 8; }   // 128 KB of shared memory

// The one-pass K / V launch with TMAX tiles per CTA and `cl` CTAs per
// cluster.  `done` stays false (and nothing is launched) when the device
// cannot place such a cluster.
template <int D, bool BF16, bool SV, int TMAX>
static cudaError_t launch_kv_cluster(const PrepassJob& j, int cl, cudaStream_t s, bool& done) {
  done = false;
  auto k = prepass_kv_cluster_kernel<D, BF16, SV, TMAX>;
  const int dyn = TMAX * kv_tile_bytes<D>();
  const int n_k = j.do_k ? j.nseq * j.Hkv : 0;
  const long long jobs = (long long)n_k + (j.do_v ? (long long)j.nseq * j.Hkv : 0);
  if (jobs == 0) {
    done = true;
    return cudaSuccess;
  }
  if (jobs * cl > 0x7fffffffLL) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e != cudaSuccess) return e;
  if (cl > 8 && (e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess)
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(jobs * cl), 1, 1);
  cfg.blockDim = dim3(kPrepassThreads, 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cl;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int fit = 0;
  if (cudaOccupancyMaxActiveClusters(&fit, k, &cfg) != cudaSuccess || fit < 1) {
    (void)cudaGetLastError();      // not placeable: the caller takes the two-launch path
    return cudaSuccess;
  }
  e = cudaLaunchKernelEx(&cfg, k, j, n_k);
  done = e == cudaSuccess;
  return e;
}

// Tiles of the longest sequence's keys -> (TMAX, cluster size) of the
// one-pass path, or false when a head does not fit a cluster.
template <int D>
static bool kv_cluster_shape(const PrepassJob& j, int& tmax, int& cl) {
  const long long tiles = j.seqs.cu_k ? ((long long)j.seqs.max_seqlen + kTile - 1) / kTile : j.seqs.tps;
  if (tiles <= 0) return false;
  for (tmax = 2; tmax <= kv_max_tiles_per_cta<D>(); tmax *= 2)
    if ((long long)kKvMaxCluster * tmax >= tiles) break;
  if (tmax > kv_max_tiles_per_cta<D>()) return false;
  const int need = (int)((tiles + tmax - 1) / tmax);
  for (cl = 1; cl < need; cl *= 2) {}
  return true;
}

template <int D, bool BF16, bool SV>
static cudaError_t launch_kv_one_pass(const PrepassJob& j, cudaStream_t s, bool& done) {
  done = false;
  int tmax = 0, cl = 0;
  if (!kv_cluster_shape<D>(j, tmax, cl)) return cudaSuccess;
  if (tmax == 2) return launch_kv_cluster<D, BF16, SV, 2>(j, cl, s, done);
  if (tmax == 4) return launch_kv_cluster<D, BF16, SV, 4>(j, cl, s, done);
  if constexpr (kv_max_tiles_per_cta<D>() >= 8) return launch_kv_cluster<D, BF16, SV, 8>(j, cl, s, done);
  return cudaSuccess;
}

template <int D, bool BF16, bool SV>
static cudaError_t launch_prepass(const PrepassJob& j0, cudaStream_t s, int* path) {
  // Launches A / B; with j0.one_pass K and V go through the cluster kernel
  // where a head fits one (it reads them once, but each CTA loads, waits at
  // the cluster barrier and then computes, and on B200 that measured slower
  // than the two launches for every workload tried).
  PrepassJob j = j0;
  if (path) *path = 0;
  if ((j0.do_k || j0.do_v) && j0.tiles_k > 0) {
    bool done = false;
    if (j0.one_pass) {
      const cudaError_t e = launch_kv_one_pass<D, BF16, SV>(j0, s, done);
      if (e != cudaSuccess) return e;
    }
    if (done) j.do_k = j.do_v = 0;
    if (path) *path = done ? kPrepassOnePass : kPrepassTwoLaunch;
  }
  const int nq = j.do_q ? j.Hq : 0;
  const int nks = (j.do_k && j.smooth_k) ? j.Hkv : 0;
  const int nvs = (j.do_v && j.pv8) ? j.Hkv : 0;
  const int xa = max(nq ? j.tiles_q : 0, (nks + nvs) ? j.tiles_k : 0);
  if (nq + nks + nvs > 0 && xa > 0) {
    prepass_a_kernel<D, BF16, SV><<<dim3(xa, nq + nks + nvs), kPrepassThreads, 0, s>>>(j);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int nb = (j.do_k ? j.Hkv : 0) + (j.do_v ? j.Hkv : 0);
  if (nb > 0 && j.tiles_k > 0) {
    prepass_b_kernel<D, BF16, SV><<<dim3(j.tiles_k, nb), kPrepassThreads, 0, s>>>(j);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (j0.q_bias && j0.do_q && j0.do_k && j0.tiles_q > 0)
    qbias_kernel<D><<<dim3(j0.tiles_q, j0.seqs.tps, j0.Hq), kTile, 0, s>>>(j0, j0.q_bias);
  return cudaGetLastError();
}

template <bool SV>
static cudaError_t prepass_dispatch(const PrepassJob& j, int D, cudaStream_t s, int* path) {
  if (D == 128)
    return j.bf16 ? launch_prepass<128, true, SV>(j, s, path) : launch_prepass<128, false, SV>(j, s, path);
  return j.bf16 ? launch_prepass<64, true, SV>(j, s, path) : launch_prepass<64, false, SV>(j, s, path);
}

cudaError_t prepass_run(const PrepassJob& j, int D, cudaStream_t s, int* path) {
  return j.smooth_v ? prepass_dispatch<true>(j, D, s, path) : prepass_dispatch<false>(j, D, s, path);
}

cudaError_t prepass_varlen_offsets(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q, int cap_k,
                                   int* toff_q, int* toff_k, uint32_t* err, cudaStream_t s) {
  varlen_offsets_kernel<<<1, 32, 0, s>>>(cu_q, cu_k, n, max_seqlen, cap_q, cap_k, toff_q, toff_k, err);
  return cudaGetLastError();
}

}  // namespace sage
