// prepass.cu -- smooth + quantize pre-pass (HBM-bound), one persistent launch.
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
// Scheduling.  The K mean and the V channel maxima need every token of a
// sequence before any K / V tile can be quantized.  One persistent kernel
// takes work items from an atomic ticket, in this order for each (sequence,
// KV head) group:
//     statistics items (K channel sums, V channel |max|, one 128-token tile each),
//     the Q tiles of the query heads that read this KV head,
//     the K tiles, the V tiles.
// A K / V tile item waits (bounded) until its group's statistics items are
// done; items are claimed in ticket order, so the items it waits for are
// already held by running CTAs.  The K / V bytes are read a second time a few
// dozen items after the statistics pass read them, while they are still in
// L2: HBM sees Q, K, V read once and the codes written once, 9 bytes per
// (token, head, channel) in FP8 mode.
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

constexpr int kStatChunk = kTile;   // tokens per statistics item (one tile)
constexpr int kPrepassThreads = 256;

// ---------------------------------------------------------------- item layout
struct ItemGeom {
  int ns, nt, per_group;   // statistics items, tiles, items per (sequence, KV head)
  int off_q, off_k, off_v; // first item of each kind within a group
};

__host__ __device__ __forceinline__ ItemGeom item_geom(const PrepassJob& j, int L) {
  ItemGeom g;
  g.nt = (L + kTile - 1) / kTile;
  const bool stats = (j.do_k && j.smooth_k) || (j.do_v && j.pv8);
  g.ns = stats ? (L + kStatChunk - 1) / kStatChunk : 0;
  g.off_q = g.ns;
  g.off_k = g.off_q + (j.do_q ? j.group * g.nt : 0);
  g.off_v = g.off_k + (j.do_k ? g.nt : 0);
  g.per_group = g.off_v + (j.do_v ? g.nt : 0);
  return g;
}

// ---------------------------------------------------------------- varlen offsets
// toff[b] = sum_{b'<b} ceil(L_b'/128) for q and k; item_off[b] = first work
// item of sequence b in the pre-pass.  Checks lengths against max_seqlen and
// the workspace's tile capacity.
__global__ void varlen_offsets_kernel(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q,
                                      int cap_k, int* toff_q, int* toff_k, uint32_t* err, PrepassJob job) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int aq = 0, ak = 0, items = 0;
  bool bad = cu_q[0] != 0 || cu_k[0] != 0;
  for (int b = 0; b < n; ++b) {
    toff_q[b] = aq;
    toff_k[b] = ak;
    job.item_off[b] = items;
    int lq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
    if (lq < 0 || lk < 0) bad = true;
    if (lq > max_seqlen || lk > max_seqlen) atomicOr(err, kErrSeqTooLong);
    lq = max(lq, 0);
    lk = max(lk, 0);
    aq += (lq + kTile - 1) / kTile;
    ak += (lk + kTile - 1) / kTile;
    // a sequence's item plan is sized by the longer of its q and k lengths
    items += job.Hkv * item_geom(job, max(lq, lk)).per_group;
  }
  toff_q[n] = aq;
  toff_k[n] = ak;
  job.item_off[n] = items;
  if (aq > cap_q || ak > cap_k) atomicOr(err, kErrTileOverflow);
  if (bad) atomicOr(err, kErrBadCuSeqlens);
}

// ---------------------------------------------------------------- statistics item
// Channel sums of K (int64 fixed point for fp16, fp64 for bf16) and channel
// |max| of V over tokens [t0, t1) (at most one tile) of one (sequence, KV
// head).  Every load of the item is issued before the first is used.
template <int D, bool BF16>
__device__ void stats_item(const PrepassJob& j, int b, int hk, int kstart, int t0, int t1, void* smem_v) {
  constexpr int TPR = D / 8, RPI = kPrepassThreads / TPR, NR = kStatChunk / RPI;
  unsigned long long(*red)[D] = reinterpret_cast<unsigned long long(*)[D]>(smem_v);
  const int cc = threadIdx.x % TPR, r0 = threadIdx.x / TPR;
  const size_t o = ((size_t)b * j.Hkv + hk) * D;
  const bool dk = j.do_k && j.smooth_k, dv = j.do_v && j.pv8;
  const uint16_t* kb = j.k + (long long)b * j.sk.sb + (long long)hk * j.sk.sh + cc * 8;
  const uint16_t* vb = j.v + (long long)b * j.sv.sb + (long long)hk * j.sv.sh + cc * 8;
  if (dk) {
    uint4 kv[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int t = t0 + r0 + RPI * i;
      kv[i] = t < t1 ? __ldg(reinterpret_cast<const uint4*>(kb + (long long)(kstart + t) * j.sk.ss))
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      // exact: fp16 as integers * 2^-24 in int64, bf16 in fp64
      long long ai = 0;
      double ad = 0.0;
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const uint16_t hv = reinterpret_cast<const uint16_t*>(&kv[i])[e];
        if (BF16) ad += (double)h16_to_f32(hv, true);
        else ai += f16_fixed24(hv);
      }
      red[r0][cc * 8 + e] = BF16 ? (unsigned long long)__double_as_longlong(ad) : (unsigned long long)ai;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kPrepassThreads) {
      if (BF16) {
        double sum = 0.0;
        for (int r = 0; r < RPI; ++r) sum += __longlong_as_double((long long)red[r][c]);
        atomicAdd(reinterpret_cast<double*>(&j.k_stat[o + c]), sum);
      } else {
        long long sum = 0;
        for (int r = 0; r < RPI; ++r) sum += (long long)red[r][c];
        atomicAdd(&j.k_stat[o + c], (unsigned long long)sum);
      }
    }
    __syncthreads();
  }
  if (dv) {
    uint4 vv[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int t = t0 + r0 + RPI * i;
      vv[i] = t < t1 ? __ldg(reinterpret_cast<const uint4*>(vb + (long long)(kstart + t) * j.sv.ss))
                     : make_uint4(0, 0, 0, 0);
    }
    float am[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const uint16_t* hv = reinterpret_cast<const uint16_t*>(&vv[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) am[e] = fmaxf(am[e], fabsf(h16_to_f32(hv[e], BF16)));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][cc * 8 + e] = __float_as_uint(am[e]);
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kPrepassThreads) {
      uint32_t m = 0;
      for (int r = 0; r < RPI; ++r) m = max(m, (uint32_t)red[r][c]);
      atomicMax(&j.v_stat[o + c], m);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- Q / K tile
template <int D, bool IS_Q, bool BF16>
__device__ void qk_tile_item(const PrepassJob& j, int b, int h, int start, int len, int toff, int tile,
                             void* smem_v) {
  constexpr int TPR = D / 8, RPI = kPrepassThreads / TPR, NR = kTile / RPI;
  struct Sm {
    double dred[RPI][D];
    float rowmax[kTile];
    float gmax[kQGroupsMax];
    float mu[D];
  };
  Sm& sm = *reinterpret_cast<Sm*>(smem_v);
  const int tg = toff + tile;
  const int tid = threadIdx.x, cc = tid % TPR, r0 = tid / TPR;
  const uint16_t* x0 = IS_Q ? j.q : j.k;
  const Strides st = IS_Q ? j.sq : j.sk;
  const uint16_t* base = x0 + (long long)b * st.sb + (long long)h * st.sh + cc * 8;
  const int H = IS_Q ? j.Hq : j.Hkv;
  const int tiles = IS_Q ? j.tiles_q : j.tiles_k;

  // raw 16-bit rows stay in registers; values are converted (and smoothed)
  // on demand in each pass
  uint4 raw[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int t = tile * kTile + r0 + RPI * i;
    raw[i] = t < len ? __ldg(reinterpret_cast<const uint4*>(base + (long long)(start + t) * st.ss))
                     : make_uint4(0, 0, 0, 0);
  }
  const int nvalid = min(kTile, len - tile * kTile);
  const bool smooth = IS_Q ? j.smooth_q : j.smooth_k;
  float mu[8] = {0, 0, 0, 0, 0, 0, 0, 0};

  if (smooth) {
    if (IS_Q) {
      // block mean: exact fp64 sum of <= 128 16-bit values per channel
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        double a = 0.0;
#pragma unroll
        for (int i = 0; i < NR; ++i) a += (double)h16_to_f32(reinterpret_cast<const uint16_t*>(&raw[i])[u], BF16);
        sm.dred[r0][cc * 8 + u] = a;
      }
      __syncthreads();
      if (tid < D) {
        double a = 0.0;
        for (int r = 0; r < RPI; ++r) a += sm.dred[r][tid];
        const float m = (float)(a / (double)nvalid);
        sm.mu[tid] = m;
        j.q_mean[((size_t)h * tiles + tg) * D + tid] = m;
      }
    } else if (tid < D) {
      // channel mean over the whole sequence from the exact sums
      const unsigned long long w = __ldcg(&j.k_stat[((size_t)b * H + h) * D + tid]);
      const double sum = BF16 ? __longlong_as_double((long long)w) : (double)(long long)w * 0x1p-24;
      const float m = (float)(sum / (double)len);
      sm.mu[tid] = m;
      if (tile == 0) j.k_mean[((size_t)b * H + h) * D + tid] = m;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u) mu[u] = sm.mu[cc * 8 + u];
  } else if (!IS_Q && tid < D && tile == 0) {
    j.k_mean[((size_t)b * H + h) * D + tid] = 0.f;
  }
  // x(i, u): the smoothed value (0 for rows past the sequence)
  auto X = [&](int i, int u) -> float {
    const int t = tile * kTile + r0 + RPI * i;
    const float v = h16_to_f32(reinterpret_cast<const uint16_t*>(&raw[i])[u], BF16);
    return t < len ? (smooth ? __fsub_rn(v, mu[u]) : v) : 0.f;
  };

  // row |max| (reduce the TPR lanes of a row), then group |max|
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) m = fmaxf(m, fabsf(X(i, u)));
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (cc == 0) sm.rowmax[r0 + RPI * i] = m;
  }
  __syncthreads();
  const int ng = IS_Q ? q_ngroups(j.gran) : k_ngroups(j.gran);
  const int warp = tid >> 5, lane = tid & 31;
  for (int g = warp; g < ng; g += kPrepassThreads / 32) {
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = lane + 32 * k;
      const int gr = IS_Q ? q_group(j.gran, r) : k_group(j.gran, r);
      if (gr == g && r < nvalid) m = fmaxf(m, sm.rowmax[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      sm.gmax[g] = m;
      float* sc = IS_Q ? j.q_scale : j.k_scale;
      sc[((size_t)h * tiles + tg) * (IS_Q ? kQGroupsMax : kKGroupsMax) + g] = __fdiv_rn(m, 127.0f);
    }
  }
  __syncthreads();

  int8_t* tbase = (IS_Q ? j.q_codes : j.k_codes) + ((size_t)h * tiles + tg) * (size_t)(kTile * D);
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = r0 + RPI * i;
    const float am = sm.gmax[IS_Q ? q_group(j.gran, r) : k_group(j.gran, r)];
    const float inv = am > 0.f ? __fdiv_rn(127.0f, am) : 0.f;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      int c = __float2int_rn(__fmul_rn(X(i, u), inv));
      c = max(-127, min(127, c));
      w[u >> 2] |= ((uint32_t)(c & 0xFF)) << ((u & 3) * 8);
    }
    *reinterpret_cast<uint2*>(tbase + swz(r, cc * 8, D)) = make_uint2(w[0], w[1]);
  }
  __syncthreads();   // the shared scratch is reused by the next item
}

// ---------------------------------------------------------------- V tile
// The 128 x D tile is staged in shared memory, then written transposed: FP8
// rows of 128 keys, or 16-bit rows split in two 64-key halves.
template <int D, bool BF16>
__device__ void v_tile_item(const PrepassJob& j, int b, int hk, int start, int len, int toff, int tile,
                            void* smem_v) {
  constexpr int TPR = D / 8, RPI = kPrepassThreads / TPR, NR = kTile / RPI;
  struct Sm {
    uint16_t vt[kTile][D];
    float inv[D];
  };
  Sm& sm = *reinterpret_cast<Sm*>(smem_v);
  const int tg = toff + tile;
  const int tid = threadIdx.x, cc = tid % TPR, r0 = tid / TPR;
  const uint16_t* base = j.v + (long long)b * j.sv.sb + (long long)hk * j.sv.sh + cc * 8;
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = r0 + RPI * i, t = tile * kTile + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < len) v = __ldg(reinterpret_cast<const uint4*>(base + (long long)(start + t) * j.sv.ss));
    *reinterpret_cast<uint4*>(&sm.vt[r][cc * 8]) = v;
  }
  if (j.pv8 && tid < D) {
    const float am = __uint_as_float(__ldcg(&j.v_stat[((size_t)b * j.Hkv + hk) * D + tid]));
    sm.inv[tid] = am > 0.f ? __fdiv_rn(kFp8Max, am) : 0.f;
    if (tile == 0) j.v_scale[((size_t)b * j.Hkv + hk) * D + tid] = __fdiv_rn(am, kFp8Max);
  }
  __syncthreads();
  uint8_t* tb = j.v_codes + ((size_t)hk * j.tiles_k + tg) * (size_t)(D * kTile * (j.pv8 ? 1 : 2));
  if (j.pv8) {
    // output chunk (channel c, keys 16k..16k+15): 16 E4M3 codes
    for (int w = tid; w < D * 8; w += kPrepassThreads) {
      const int c = w % D, k = w / D;
      const float inv = sm.inv[c];
      uint32_t o[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float f[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __fmul_rn(h16_to_f32(sm.vt[16 * k + 4 * q4 + i][c], BF16), inv);
        o[q4] = pack_e4m3x4(f[0], f[1], f[2], f[3]);
      }
      *reinterpret_cast<uint4*>(tb + swz(c, 16 * k, 128)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    // output chunk (half hf, channel c, keys 64hf + 8kk .. +7): 8 16-bit values
    for (int w = tid; w < D * 16; w += kPrepassThreads) {
      const int c = w % D, k = w / D, hf = k >> 3, kk = k & 7;
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = 64 * hf + 8 * kk + 2 * i;
        o[i] = (uint32_t)sm.vt[key][c] | ((uint32_t)sm.vt[key + 1][c] << 16);
      }
      *reinterpret_cast<uint4*>(tb + (size_t)hf * (D * 128) + swz(c, 16 * kk, 128)) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
}

// Bounded wait for a group's statistics items (K sums / V maxima).
__device__ __forceinline__ bool wait_stats(const PrepassJob& j, int g, int ns, int* flag_s) {
  if (threadIdx.x == 0) {
    int ok = 1;
    if (ns > 0) {
      const uint64_t t0 = global_timer_ns();
      while (atomicAdd(&j.stats_done[g], 0u) < (uint32_t)ns) {
        __nanosleep(256);
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          atomicOr(j.err, kErrTimeoutPrepass);
          ok = 0;
          break;
        }
      }
      __threadfence();
    }
    *flag_s = ok;
  }
  __syncthreads();
  const bool ok = *flag_s != 0;
  __syncthreads();
  return ok;
}

// ---------------------------------------------------------------- the kernel
template <int D>
struct PrepassSmem {
  static constexpr int V = kTile * D * 2 + D * 4;
  static constexpr int QK = (kPrepassThreads / (D / 8)) * D * 8 + kTile * 4 + kQGroupsMax * 4 + D * 4;
  static constexpr int ST = (kPrepassThreads / (D / 8)) * D * 8;
  static constexpr int BYTES = V > QK ? (V > ST ? V : ST) : (QK > ST ? QK : ST);
};

template <int D, bool BF16>
__global__ void __launch_bounds__(kPrepassThreads, 3) prepass_kernel(PrepassJob j) {
  __shared__ __align__(16) uint8_t smem[PrepassSmem<D>::BYTES];
  __shared__ int item_s, flag_s;
  const bool varlen = j.seqs.cu_k != nullptr;
  const int total = varlen ? j.item_off[j.nseq] : j.nseq * j.Hkv * item_geom(j, j.seqs.S).per_group;
  for (;;) {
    if (threadIdx.x == 0) item_s = (int)atomicAdd(j.ticket, 1u);
    __syncthreads();
    const int item = item_s;
    __syncthreads();
    if (item >= total) break;
    // decode: sequence, KV head, kind
    int b, local;
    if (varlen) {
      int lo = 0, hi = j.nseq - 1;             // last b with item_off[b] <= item
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (j.item_off[mid] <= item) lo = mid;
        else hi = mid - 1;
      }
      b = lo;
      local = item - j.item_off[b];
    } else {
      const int per_seq = j.Hkv * item_geom(j, j.seqs.S).per_group;
      b = item / per_seq;
      local = item - b * per_seq;
    }
    int qs, Lq, tq0, ks, Lk, tk0;
    j.seqs.q(b, qs, Lq, tq0);
    j.seqs.k(b, ks, Lk, tk0);
    if (varlen && (Lq < 0 || Lk < 0 || Lq > j.seqs.max_seqlen || Lk > j.seqs.max_seqlen)) continue;
    const ItemGeom gp = item_geom(j, max(Lq, Lk));   // the plan of this sequence
    const ItemGeom gk = item_geom(j, Lk);            // statistics items that carry data
    const int hk = local / gp.per_group;
    const int r = local - hk * gp.per_group;
    const int g = b * j.Hkv + hk;
    if (r < gp.off_q) {                              // statistics
      const int t0 = r * kStatChunk;
      if (t0 < Lk) stats_item<D, BF16>(j, b, hk, ks, t0, min(Lk, t0 + kStatChunk), smem);
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(&j.stats_done[g], 1u);
      }
    } else if (r < gp.off_k) {                       // Q tile
      const int hl = (r - gp.off_q) / gp.nt, tile = (r - gp.off_q) % gp.nt;
      if (tile * kTile < Lq && tq0 + tile < j.tiles_q)
        qk_tile_item<D, true, BF16>(j, b, hk * j.group + hl, qs, Lq, tq0, tile, smem);
    } else if (r < gp.off_v) {                       // K tile
      const int tile = r - gp.off_k;
      if (wait_stats(j, g, j.smooth_k ? gp.ns : 0, &flag_s) && tile * kTile < Lk && tk0 + tile < j.tiles_k)
        qk_tile_item<D, false, BF16>(j, b, hk, ks, Lk, tk0, tile, smem);
    } else {                                         // V tile
      const int tile = r - gp.off_v;
      if (wait_stats(j, g, j.pv8 ? gp.ns : 0, &flag_s) && tile * kTile < Lk && tk0 + tile < j.tiles_k)
        v_tile_item<D, BF16>(j, b, hk, ks, Lk, tk0, tile, smem);
    }
    (void)gk;
  }
}

// ---------------------------------------------------------------- launchers
template <int D, bool BF16>
static cudaError_t launch_prepass(const PrepassJob& j, cudaStream_t s) {
  int dev = 0, num_sms = 0, bps = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, prepass_kernel<D, BF16>, kPrepassThreads, 0);
  if (e != cudaSuccess) return e;
  prepass_kernel<D, BF16><<<max(1, num_sms * max(1, bps)), kPrepassThreads, 0, s>>>(j);
  return cudaGetLastError();
}

cudaError_t prepass_run(const PrepassJob& j, int D, cudaStream_t s) {
  if (D == 128) return j.bf16 ? launch_prepass<128, true>(j, s) : launch_prepass<128, false>(j, s);
  return j.bf16 ? launch_prepass<64, true>(j, s) : launch_prepass<64, false>(j, s);
}

cudaError_t prepass_varlen_offsets(const int* cu_q, const int* cu_k, int n, int max_seqlen, int cap_q, int cap_k,
                                   int* toff_q, int* toff_k, uint32_t* err, const PrepassJob& job,
                                   cudaStream_t s) {
  varlen_offsets_kernel<<<1, 32, 0, s>>>(cu_q, cu_k, n, max_seqlen, cap_q, cap_k, toff_q, toff_k, err, job);
  return cudaGetLastError();
}

}  // namespace sage
