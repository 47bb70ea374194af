// attn_fwd.cu -- quantized attention forward on sm_100a tensor cores.
//
// Method (SageAttention2 summary, sgqg.cn, sections 相关工作 and
// SageAttention2方法; Kairos SageAttention page, sections 2.1-2.2):
// FlashAttention tiling over 128-key tiles; S = Q_i8 K_i8^T on the INT8 tensor
// cores with int32 accumulation, dequantized with the Q/K group scales; online
// softmax with exp2; P~ (<= 1 after max subtraction) rounded to E4M3 with the
// static scale 448 and multiplied with per-channel E4M3 V on the FP8 tensor
// cores (or P~ and V in 16 bits); the partial sums either accumulate in one
// FP32 tensor-memory accumulator (fp32) or, per tile, into a separate FP32
// register accumulator (fp32+fp32, the two-level scheme).
//
// B200 design.  One CTA owns NQ query tiles of 128 rows of one (sequence,
// head) and runs four roles:
//   warp 0        loader: one bulk copy per MMA-ready tile (the pre-pass wrote
//                 tiles already in the swizzled operand layout), NST stages;
//   warp 1        MMA issuer: tcgen05.mma kind::i8 (S, SMEM x SMEM -> TMEM s32)
//                 and kind::f8f6f4 / kind::f16 (O, P~ from TMEM x V from SMEM);
//   warp 2        tensor-memory allocation;
//   WG 1..NQ      softmax, one thread per query row (TMEM lane): integer row
//                 max per scale group, one FFMA + ex2 per score, P~ packed and
//                 written back into TMEM over the S it came from;
//   last WG       correction: rescales O in TMEM (fp32) or adds the per-tile
//                 partial O into FP32 registers (fp32+fp32); epilogue.
// Every mbarrier wait is bounded (sage_common.cuh): a wait that never ends sets
// the device error word and the CTA tears down instead of hanging.
#include "sage_launch.cuh"

namespace sage {

template <int D, bool PV8, bool ACC2>
struct AttnCfg {
  static constexpr int NQ = ACC2 ? 1 : 2;          // query tiles per CTA
  static constexpr int NSB = ACC2 ? 2 : 1;         // S buffers per query tile
  static constexpr int NST = 3;                    // K/V pipeline stages
  static constexpr int NTHREADS = 384;             // 3 warpgroups (168 registers per thread)
  static constexpr int QT = kTile * D;             // bytes of a Q or K tile
  static constexpr int VT = D * kTile * (PV8 ? 1 : 2);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * QT;
  static constexpr int OFF_V = OFF_K + NST * QT;
  static constexpr int OFF_ALPHA = OFF_V + NST * VT;          // float [NQ][2][128]   (two-level)
  static constexpr int OFF_L = OFF_ALPHA + NQ * 2 * 128 * 4;  // float [NQ][128]      (two-level)
  static constexpr int OFF_BAR = OFF_L + NQ * 128 * 4;
  enum {
    B_QFULL = 0,
    B_KFULL = B_QFULL + NQ,
    B_KEMPTY = B_KFULL + NST,
    B_VFULL = B_KEMPTY + NST,
    B_VEMPTY = B_VFULL + NST,
    B_SFULL = B_VEMPTY + NST,
    B_PFULL = B_SFULL + NQ * NSB,    // softmax -> MMA: P~ in TMEM (and O rescaled)
    B_OFULL = B_PFULL + NQ,          // MMA -> consumer of O (every PV two-level, last PV one-level)
    B_OREADY = B_OFULL + NQ,         // correction -> MMA: partial O consumed (two-level)
    B_AFULL = B_OREADY + NQ,         // softmax -> correction: alpha (two-level)
    B_AEMPTY = B_AFULL + 2 * NQ,
    B_LFULL = B_AEMPTY + 2 * NQ,     // softmax -> correction: final row sum (two-level)
    B_DONE = B_LFULL + NQ,
    NBAR = B_DONE + 1
  };
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // [0] tmem base, [1] abort flag
  static constexpr int SMEM_USED = OFF_MISC + 16;
  // At least 116 KB so that a single CTA holds an SM: the CTA allocates all
  // 512 TMEM columns, a second resident CTA would only wait for them.
  static constexpr int SMEM_BYTES = (SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024) + 1024;
  static constexpr int TM_S = 0;                   // S[q][b] at (q*NSB + b) * 128
  static constexpr int TM_O = NQ * NSB * 128;      // O[q] at TM_O + q * D
  static constexpr uint32_t TM_COLS = 512;
  static_assert(TM_O + NQ * D <= 512, "TMEM budget");
  static_assert(SMEM_USED + 1024 <= 227 * 1024, "shared memory budget");
};

// ---------------------------------------------------------------- softmax
// KPT: per-thread K groups ((col/64)*8 + col%8), else per-64-key groups.
template <bool KPT>
__device__ __forceinline__ constexpr int kgrp(int col) {
  return KPT ? ((col >> 6) << 3) + (col & 7) : (col >> 6);
}

// One 128-key tile of one query row (this thread's TMEM lane):
//   S (int32, TMEM) -> exact float (magic-number add) -> group maxima of the
//   unscaled scores -> m_tile = max_g c_g * max_g(S) -> alpha -> exponent
//   argument S*c - m (one packed FFMA), ex2, row sum -> P~ rounded to E4M3
//   (448 folded into the exponent) or 16 bits, written over the S columns.
// c[g] = dQ * dK_g * sm_scale * log2(e), kept >= 1e-30 so that a masked
// score (-inf) always yields P~ = 0 (a group whose scale is 0 has S = 0 and
// s = S * 1e-30 rounds every P~ exactly as s = 0 does).
template <bool PV8, bool KPT, bool BF16P>
__device__ __forceinline__ void softmax_tile(uint32_t taddr, const float (&c)[16], bool masked, int col0, int lim,
                                             float& m, float& l, float& alpha) {
  uint32_t r[128];
  tmem_ld128_sync(taddr, r);
#pragma unroll
  for (int k = 0; k < 64; ++k) {
    float x0, x1;
    add2(x0, x1, __uint_as_float(r[2 * k] + 0x4B400000u), __uint_as_float(r[2 * k + 1] + 0x4B400000u),
         -12582912.0f, -12582912.0f);
    r[2 * k] = __float_as_uint(x0);
    r[2 * k + 1] = __float_as_uint(x1);
  }
  if (masked) {
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if (!(col0 + i < lim)) r[i] = 0xFF800000u;   // -inf
  }
  auto F = [&](int i) { return __uint_as_float(r[i]); };
  // maxima of the unscaled scores per scale group (c > 0 keeps the order)
  float mt = -INFINITY;
  if (KPT) {
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      const int base = (g >> 3) * 64 + (g & 7);
      float a = max3(F(base), F(base + 8), F(base + 16));
      float bb = max3(F(base + 24), F(base + 32), F(base + 40));
      a = max3(a, bb, fmaxf(F(base + 48), F(base + 56)));
      mt = fmaxf(mt, c[g] * a);
    }
  } else {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; i += 8) {
        a0 = max3(a0, F(64 * g + i), F(64 * g + i + 1));
        a1 = max3(a1, F(64 * g + i + 2), F(64 * g + i + 3));
        a2 = max3(a2, F(64 * g + i + 4), F(64 * g + i + 5));
        a3 = max3(a3, F(64 * g + i + 6), F(64 * g + i + 7));
      }
      mt = fmaxf(mt, c[g] * max3(a0, a1, fmaxf(a2, a3)));
    }
  }
  const float m_new = fmaxf(m, mt);
  alpha = (m == -INFINITY) ? 0.f : ex2(m - m_new);
  const float nb = -(PV8 ? (m_new - kLog2Fp8Max) : m_new);
  float ls0 = 0.f, ls1 = 0.f, h0 = 0.f, h1 = 0.f;
  uint32_t w[PV8 ? 32 : 64];
#pragma unroll
  for (int k = 0; k < 64; ++k) {
    float a0, a1;
    fma2(a0, a1, F(2 * k), F(2 * k + 1), c[kgrp<KPT>(2 * k)], c[kgrp<KPT>(2 * k + 1)], nb, nb);
    const float p0 = ex2(a0), p1 = ex2(a1);
    add2(ls0, ls1, ls0, ls1, p0, p1);
    if (PV8) {
      if (k & 1) w[k >> 1] = pack_e4m3x4(h0, h1, p0, p1);
      else { h0 = p0; h1 = p1; }
    } else {
      w[k] = BF16P ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
    }
  }
  l = alpha * l + (ls0 + ls1);
  m = m_new;
  if (PV8) {
    tmem_st32(taddr, reinterpret_cast<const uint32_t(&)[32]>(w[0]));
  } else {
    tmem_st32(taddr, reinterpret_cast<const uint32_t(&)[32]>(w[0]));
    tmem_st32(taddr + 32, reinterpret_cast<const uint32_t(&)[32]>(w[PV8 ? 0 : 32]));
  }
}

// Row epilogue: out[c] = O[c] * inv_l (* delta_V[c] in FP8 mode, where l sums
// 448 * P~ and O sums P8 * V8, so the 448 cancels); 16-bit rounding, one row.
template <int D, bool PV8, bool FROM_REGS>
__device__ __forceinline__ void store_row(uint16_t* orow, uint32_t ob, const float* oacc, float inv_l,
                                          const float* vsc, bool bf16, bool have_o, bool valid) {
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    float o[32];
    if (FROM_REGS) {
#pragma unroll
      for (int u = 0; u < 32; ++u) o[u] = oacc[ch * 32 + u];
    } else {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32(ob + ch * 32, r);
        tmem_wait_ld(r);
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) o[u] = have_o ? __uint_as_float(r[u]) : 0.f;
    }
    uint32_t w[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a = o[2 * k] * inv_l, bb = o[2 * k + 1] * inv_l;
      if (PV8) {
        a *= __ldg(vsc + ch * 32 + 2 * k);
        bb *= __ldg(vsc + ch * 32 + 2 * k + 1);
      }
      w[k] = bf16 ? pack_bf16x2(a, bb) : pack_f16x2(a, bb);
    }
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
  }
}

// One softmax warpgroup: the online softmax of query tile q over its KV
// tiles; in one-level mode also the O rescale and the epilogue.
template <int D, bool PV8, bool ACC2, bool KPT, bool BF16P>
__device__ __forceinline__ void softmax_role(const AttnParams& p, uint32_t sb, uint32_t tmem, int warp, int tid,
                                             int pair, int b, int h, int hk, int qs, int Lq, int Lk, int tq0,
                                             int tk0, const int* n, const float* vsc) {
  using C = AttnCfg<D, PV8, ACC2>;
  constexpr int NQ = C::NQ, NSB = C::NSB;
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  uint8_t* smem = reinterpret_cast<uint8_t*>(__cvta_shared_to_generic(sb));
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* alpha_s = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  float* l_s = reinterpret_cast<float*>(smem + C::OFF_L);
    const int q = (warp - 4) >> 2;
    const int t = tid - 128 * (1 + q);
    const int qt = pair * NQ + q;
    const uint32_t lane_off = (uint32_t)((t & ~31)) << 16;
    const int row = qt * kTile + t;
    const bool bf16 = BF16P || (PV8 && p.out_bf16 != 0);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (n[q] > 0) {
      const float qsc = p.q_scale[((size_t)h * p.tiles_q + tq0 + qt) * kQGroupsMax + q_group(p.gran, t)];
      const float* ksb = p.k_scale + ((size_t)hk * p.tiles_k + tk0) * kKGroupsMax;
      const uint32_t ob = tmem + C::TM_O + q * D + lane_off;
      // K group scales of the next tile are fetched one tile ahead
      float ksn[KPT ? 16 : 2];
#pragma unroll
      for (int g = 0; g < (KPT ? 16 : 2); ++g) ksn[g] = __ldg(ksb + g);
      for (int j = 0; j < n[q]; ++j) {
        const int buf = j % NSB;
        float c[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) c[g] = g < (KPT ? 16 : 2) ? fmaxf((qsc * ksn[g]) * p.sl2, 1e-30f) : 1e-30f;
        if (j + 1 < n[q]) {
#pragma unroll
          for (int g = 0; g < (KPT ? 16 : 2); ++g) ksn[g] = __ldg(ksb + (j + 1) * kKGroupsMax + g);
        }
        if (!(ok = mbar_wait(bar(C::B_SFULL + q * NSB + buf), (j / NSB) & 1, abort_flag, p.err, kErrTimeoutSoftmax)))
          break;
        tc_fence_after();
        // keys past the sequence, or (causal) past this row, are masked
        const int col0 = j * kTile;
        const bool masked = (col0 + kTile > Lk) || (p.causal && j == qt);
        const int lim = p.causal ? min(Lk, row + 1) : Lk;
        const uint32_t taddr = tmem + C::TM_S + (q * NSB + buf) * 128 + lane_off;
        float alpha;
        softmax_tile<PV8, KPT, BF16P>(taddr, c, masked, col0, lim, m, l, alpha);
        if (ACC2) {
          const int ab = j & 1;
          if (!(ok = mbar_wait(bar(C::B_AEMPTY + 2 * q + ab), ((j >> 1) & 1) ^ 1, abort_flag, p.err,
                               kErrTimeoutSoftmax)))
            break;
          alpha_s[(q * 2 + ab) * 128 + t] = alpha;
          mbar_arrive(bar(C::B_AFULL + 2 * q + ab));
        } else if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O(q) holds the sums of tiles < j (PV_{j-1} finished before S_j did)
          if (D == 128) {
            uint32_t r[128];
            tmem_ld128_sync(ob, r);
#pragma unroll
            for (int u = 0; u < 128; u += 2) {
              float x0, x1;
              mul2(x0, x1, __uint_as_float(r[u]), __uint_as_float(r[u + 1]), alpha, alpha);
              r[u] = __float_as_uint(x0);
              r[u + 1] = __float_as_uint(x1);
            }
            tmem_st128(ob, r);
          } else {
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t r[32];
              tmem_ld32(ob + ch * 32, r);
              tmem_wait_ld(r);
#pragma unroll
              for (int u = 0; u < 32; u += 2) {
                float x0, x1;
                mul2(x0, x1, __uint_as_float(r[u]), __uint_as_float(r[u + 1]), alpha, alpha);
                r[u] = __float_as_uint(x0);
                r[u + 1] = __float_as_uint(x1);
              }
              tmem_st32(ob + ch * 32, r);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + q));
      }
    }
    if (ACC2) {
      l_s[q * 128 + t] = l;
      mbar_arrive(bar(C::B_LFULL + q));
    } else if (ok && qt * kTile < Lq) {
      // epilogue of this query tile
      if (n[q] > 0) {
        ok = mbar_wait(bar(C::B_OFULL + q), 0, abort_flag, p.err, kErrTimeoutSoftmax);
        tc_fence_after();
      }
      if (ok) {
        uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + (long long)b * p.os.sb + (long long)h * p.os.sh +
                         (long long)(qs + row) * p.os.ss;
        store_row<D, PV8, false>(orow, tmem + C::TM_O + q * D + lane_off, nullptr, l > 0.f ? 1.0f / l : 0.f, vsc,
                                 bf16, n[q] > 0, row < Lq);
      }
    }
}

// ---------------------------------------------------------------- kernel
// Warp roles: 0 loader, 1 MMA issuer, 2 TMEM allocator, 3 idle; warpgroups
// 1..NQ softmax (one query tile each).  One-level accumulation: the softmax
// warpgroup also rescales O in TMEM (before releasing P~ to the MMA) and runs
// the epilogue.  Two-level: warpgroup 2 is the correction warpgroup holding
// the FP32 outer accumulator in registers.
template <int D, bool PV8, bool ACC2>
__global__ void __launch_bounds__(384, 1) attn_fwd_kernel(const AttnParams p) {
  using C = AttnCfg<D, PV8, ACC2>;
  constexpr int NQ = C::NQ, NSB = C::NSB, NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* alpha_s = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  float* l_s = reinterpret_cast<float*>(smem + C::OFF_L);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int pair = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  int qs, Lq, tq0, ks, Lk, tk0;
  p.seqs.q(b, qs, Lq, tq0);
  p.seqs.k(b, ks, Lk, tk0);
  if (p.seqs.cu_q && (Lq > p.seqs.max_seqlen || Lk > p.seqs.max_seqlen || Lq < 0 || Lk < 0)) return;
  if (pair * NQ * kTile >= Lq) return;             // uniform: before any setup
  const int hk = h / p.group;
  const int nk = (Lk + kTile - 1) / kTile;
  int n[NQ];
  int maxn = 0;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int qt = pair * NQ + q;
    const bool valid = qt * kTile < Lq;
    n[q] = !valid ? 0 : (p.causal ? min(nk, qt + 1) : nk);
    maxn = max(maxn, n[q]);
  }
  // the workspace must hold every tile this CTA reads (varlen: the offsets
  // kernel has already flagged an overflow)
  if (tq0 + (Lq + kTile - 1) / kTile > p.tiles_q || tk0 + nk > p.tiles_k) return;

  if (tid == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      uint32_t cnt = 1;
      if ((i >= C::B_PFULL && i < C::B_PFULL + NQ) || (i >= C::B_OREADY && i < C::B_OREADY + NQ) ||
          (i >= C::B_AFULL && i < C::B_AFULL + 4 * NQ) || (i >= C::B_LFULL && i < C::B_LFULL + NQ))
        cnt = 128;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(misc), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const float* vsc = p.v_scale + ((size_t)b * p.Hkv + hk) * D;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      const int8_t* qb = p.q_codes + ((size_t)h * p.tiles_q + tq0 + pair * NQ) * C::QT;
      for (int q = 0; q < NQ; ++q)
        if (n[q] > 0) {
          mbar_expect_tx(bar(C::B_QFULL + q), C::QT);
          bulk_g2s(sb + C::OFF_Q + q * C::QT, qb + (size_t)q * C::QT, C::QT, bar(C::B_QFULL + q));
        }
      const int8_t* kb = p.k_codes + ((size_t)hk * p.tiles_k + tk0) * C::QT;
      const uint8_t* vb = p.v_codes + ((size_t)hk * p.tiles_k + tk0) * (size_t)C::VT;
      int issued_k = 0, issued_v = 0;
      for (int t = 0; t < maxn; ++t) {
        const int st = t % NST, u = t / NST;
        if (u > 0 && !mbar_wait(bar(C::B_KEMPTY + st), (u - 1) & 1, abort_flag, p.err, kErrTimeoutLoad)) break;
        mbar_expect_tx(bar(C::B_KFULL + st), C::QT);
        bulk_g2s(sb + C::OFF_K + st * C::QT, kb + (size_t)t * C::QT, C::QT, bar(C::B_KFULL + st));
        issued_k = t + 1;
        if (u > 0 && !mbar_wait(bar(C::B_VEMPTY + st), (u - 1) & 1, abort_flag, p.err, kErrTimeoutLoad)) break;
        mbar_expect_tx(bar(C::B_VFULL + st), C::VT);
        bulk_g2s(sb + C::OFF_V + st * C::VT, vb + (size_t)t * C::VT, C::VT, bar(C::B_VFULL + st));
        issued_v = t + 1;
      }
      if (*abort_flag) {
        // let copies in flight land before the CTA's shared memory is released
        for (int t = max(0, issued_k - NST); t < issued_k; ++t) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(C::B_KFULL + t % NST), (t / NST) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
        for (int t = max(0, issued_v - NST); t < issued_v; ++t) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(C::B_VFULL + t % NST), (t / NST) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
        for (int q = 0; q < NQ; ++q)
          if (n[q] > 0) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::B_QFULL + q), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && maxn > 0) {
      constexpr uint32_t ID_QK = idesc_i8(128, 128);
      const uint32_t ID_PV = PV8 ? idesc_e4m3(128, D) : idesc_f16(128, D, p.out_bf16 != 0);
      bool ok = true;
      for (int q = 0; q < NQ && ok; ++q)
        if (n[q] > 0) ok = mbar_wait(bar(C::B_QFULL + q), 0, abort_flag, p.err, kErrTimeoutMma);
      tc_fence_after();
      auto mma_s = [&](int q, int t, int st) {
        const uint32_t d = tmem + C::TM_S + (q * NSB + t % NSB) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t a = smem_desc(sb + C::OFF_Q + q * C::QT + kk * 32, D);
          const uint64_t bd = smem_desc(sb + C::OFF_K + st * C::QT + kk * 32, D);
          mma_i8_ss(d, a, bd, ID_QK, kk > 0);
        }
        tc_commit(bar(C::B_SFULL + q * NSB + t % NSB));
      };
      auto mma_pv = [&](int q, int j, int st) {
        const uint32_t a0 = tmem + C::TM_S + (q * NSB + j % NSB) * 128;
        const uint32_t d = tmem + C::TM_O + q * D;
        if (PV8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ts(d, a0 + kk * 8, smem_desc(sb + C::OFF_V + st * C::VT + kk * 32, 128), ID_PV,
                      ACC2 ? (kk > 0) : (j > 0 || kk > 0));
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ts(d, a0 + kk * 8,
                       smem_desc(sb + C::OFF_V + st * C::VT + (kk >> 2) * (D * 128) + (kk & 3) * 32, 128), ID_PV,
                       ACC2 ? (kk > 0) : (j > 0 || kk > 0));
        }
      };
      // S for the first NSB tiles
      for (int t = 0; t < NSB && t < maxn && ok; ++t) {
        ok = mbar_wait(bar(C::B_KFULL + t % NST), (t / NST) & 1, abort_flag, p.err, kErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        for (int q = 0; q < NQ; ++q)
          if (t < n[q]) mma_s(q, t, t % NST);
        tc_commit(bar(C::B_KEMPTY + t % NST));
      }
      for (int j = 0; j < maxn && ok; ++j) {
        const int st = j % NST, t = j + NSB;
        if (!(ok = mbar_wait(bar(C::B_VFULL + st), (j / NST) & 1, abort_flag, p.err, kErrTimeoutMma))) break;
        bool kready = false;
        for (int q = 0; q < NQ && ok; ++q) {
          if (j < n[q]) {
            ok = mbar_wait(bar(C::B_PFULL + q), j & 1, abort_flag, p.err, kErrTimeoutMma);
            if (ok && ACC2 && j > 0)
              ok = mbar_wait(bar(C::B_OREADY + q), (j - 1) & 1, abort_flag, p.err, kErrTimeoutMma);
            if (!ok) break;
            tc_fence_after();
            mma_pv(q, j, st);
            if (ACC2 || j == n[q] - 1) tc_commit(bar(C::B_OFULL + q));
          }
          if (t < n[q]) {
            if (!kready) {
              if (!(ok = mbar_wait(bar(C::B_KFULL + t % NST), (t / NST) & 1, abort_flag, p.err, kErrTimeoutMma)))
                break;
              tc_fence_after();
              kready = true;
            }
            mma_s(q, t, t % NST);
          }
        }
        if (!ok) break;
        tc_commit(bar(C::B_VEMPTY + st));
        if (kready) tc_commit(bar(C::B_KEMPTY + t % NST));
      }
      // all MMAs issued by this thread complete before teardown
      tc_commit(bar(C::B_DONE));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(C::B_DONE), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
    }
  } else if (warp >= 4 && warp < 4 + 4 * NQ) {
    // ------------------------------------------------------------ softmax
    const bool bf16p = !PV8 && p.out_bf16;
    if (p.gran == 2) {
      if (bf16p) softmax_role<D, PV8, ACC2, true, true>(p, sb, tmem, warp, tid, pair, b, h, hk, qs, Lq, Lk, tq0, tk0, n, vsc);
      else softmax_role<D, PV8, ACC2, true, false>(p, sb, tmem, warp, tid, pair, b, h, hk, qs, Lq, Lk, tq0, tk0, n, vsc);
    } else {
      if (bf16p) softmax_role<D, PV8, ACC2, false, true>(p, sb, tmem, warp, tid, pair, b, h, hk, qs, Lq, Lk, tq0, tk0, n, vsc);
      else softmax_role<D, PV8, ACC2, false, false>(p, sb, tmem, warp, tid, pair, b, h, hk, qs, Lq, Lk, tq0, tk0, n, vsc);
    }
  } else if (ACC2 && warp >= 4 + 4 * NQ) {
    // ------------------------------------------------------------ correction (two-level) + epilogue
    const int t = tid - 128 * (1 + NQ);
    const uint32_t lane_off = (uint32_t)((t & ~31)) << 16;
    const uint32_t ob = tmem + C::TM_O + lane_off;
    bool ok = true;
    float oacc[D];
#pragma unroll
    for (int i = 0; i < D; ++i) oacc[i] = 0.f;
    for (int j = 0; j < n[0] && ok; ++j) {
      const int ab = j & 1;
      if (!(ok = mbar_wait(bar(C::B_AFULL + ab), (j >> 1) & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
      const float alpha = alpha_s[ab * 128 + t];
      mbar_arrive(bar(C::B_AEMPTY + ab));
      if (!(ok = mbar_wait(bar(C::B_OFULL), j & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < D / 16; ++ch) {
        uint32_t r[16];
        tmem_ld16(ob + ch * 16, r);
        tmem_wait_ld(r);
#pragma unroll
        for (int u = 0; u < 16; u += 2)
          fma2(oacc[ch * 16 + u], oacc[ch * 16 + u + 1], alpha, alpha, oacc[ch * 16 + u], oacc[ch * 16 + u + 1],
               __uint_as_float(r[u]), __uint_as_float(r[u + 1]));
      }
      tc_fence_before();
      mbar_arrive(bar(C::B_OREADY));
    }
    const int row = pair * kTile + t;
    if (ok && pair * kTile < Lq) {
      float l = 0.f;
      if (n[0] > 0) {
        ok = mbar_wait(bar(C::B_LFULL), 0, abort_flag, p.err, kErrTimeoutCorr);
        l = l_s[t];
      }
      if (ok) {
        uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + (long long)b * p.os.sb + (long long)h * p.os.sh +
                         (long long)(qs + row) * p.os.ss;
        store_row<D, PV8, true>(orow, ob, oacc, l > 0.f ? 1.0f / l : 0.f, vsc, p.out_bf16 != 0, true, row < Lq);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ---------------------------------------------------------------- debug S tile
// S = Q_tile * K_tile^T through the same descriptors / MMA as the kernel.
__global__ void __launch_bounds__(128, 1) qk_tile_kernel(const int8_t* qt, const int8_t* kt, int D,
                                                         int32_t* out, uint32_t* err) {
  __shared__ __align__(1024) uint8_t sq[kTile * 128];
  __shared__ __align__(1024) uint8_t sk[kTile * 128];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tslot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t bytes = kTile * D;
  if (tid == 0) {
    mbar_expect_tx(smem_u32(&bars[0]), 2 * bytes);
    bulk_g2s(smem_u32(sq), qt, bytes, smem_u32(&bars[0]));
    bulk_g2s(smem_u32(sk), kt, bytes, smem_u32(&bars[0]));
    if (mbar_wait(smem_u32(&bars[0]), 0, &abort_flag, err, kErrTimeoutMma)) {
      tc_fence_after();
      for (int kk = 0; kk < D / 32; ++kk)
        mma_i8_ss(tmem, smem_desc(smem_u32(sq) + kk * 32, D), smem_desc(smem_u32(sk) + kk * 32, D),
                  idesc_i8(128, 128), kk > 0);
    }
    tc_commit(smem_u32(&bars[1]));
  }
  __syncwarp();
  const bool ok = mbar_wait(smem_u32(&bars[1]), 0, &abort_flag, err, kErrTimeoutMma);
  tc_fence_after();
  if (ok) {
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + ch * 32, r);
      tmem_wait_ld(r);
#pragma unroll
      for (int u = 0; u < 32; ++u) out[tid * 128 + ch * 32 + u] = (int32_t)r[u];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------- launchers
template <int D, bool PV8, bool ACC2>
static cudaError_t launch_attn(const AttnParams& p, int n_pairs_x, int nseq, cudaStream_t s) {
  using C = AttnCfg<D, PV8, ACC2>;
  auto k = attn_fwd_kernel<D, PV8, ACC2>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  k<<<dim3(n_pairs_x, p.Hq, nseq), C::NTHREADS, C::SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

// Query tiles per CTA for a configuration (the host sizes the grid with it).
int attn_tiles_per_cta(int D, bool pv8, bool acc2) {
  (void)D; (void)pv8;
  return acc2 ? 1 : 2;
}

cudaError_t attn_forward(const AttnParams& p, int D, bool pv8, bool acc2, int max_len_q, int nseq,
                         cudaStream_t s) {
  const int per = attn_tiles_per_cta(D, pv8, acc2) * kTile;
  const int nx = (max_len_q + per - 1) / per;
  if (nx == 0 || nseq == 0) return cudaSuccess;
  if (D == 128) {
    if (pv8) return acc2 ? launch_attn<128, true, true>(p, nx, nseq, s) : launch_attn<128, true, false>(p, nx, nseq, s);
    return acc2 ? launch_attn<128, false, true>(p, nx, nseq, s) : launch_attn<128, false, false>(p, nx, nseq, s);
  }
  if (pv8) return acc2 ? launch_attn<64, true, true>(p, nx, nseq, s) : launch_attn<64, true, false>(p, nx, nseq, s);
  return acc2 ? launch_attn<64, false, true>(p, nx, nseq, s) : launch_attn<64, false, false>(p, nx, nseq, s);
}

cudaError_t debug_qk_tile(const int8_t* qt, const int8_t* kt, int D, int32_t* out, uint32_t* err,
                          cudaStream_t s) {
  qk_tile_kernel<<<1, 128, 0, s>>>(qt, kt, D, out, err);
  return cudaGetLastError();
}

}  // namespace sage
