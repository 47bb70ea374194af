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
  static constexpr int NTHREADS = (NQ + 2) * 128;
  static constexpr int QT = kTile * D;             // bytes of a Q or K tile
  static constexpr int VT = D * kTile * (PV8 ? 1 : 2);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * QT;
  static constexpr int OFF_V = OFF_K + NST * QT;
  static constexpr int OFF_ALPHA = OFF_V + NST * VT;          // float [NQ][2][128]
  static constexpr int OFF_L = OFF_ALPHA + NQ * 2 * 128 * 4;  // float [NQ][128]
  static constexpr int OFF_BAR = OFF_L + NQ * 128 * 4;
  enum {
    B_QFULL = 0,
    B_KFULL = B_QFULL + NQ,
    B_KEMPTY = B_KFULL + NST,
    B_VFULL = B_KEMPTY + NST,
    B_VEMPTY = B_VFULL + NST,
    B_SFULL = B_VEMPTY + NST,
    B_PFULL = B_SFULL + NQ * NSB,
    B_OFULL = B_PFULL + NQ,
    B_OREADY = B_OFULL + NQ,
    B_AFULL = B_OREADY + NQ,
    B_AEMPTY = B_AFULL + 2 * NQ,
    B_LFULL = B_AEMPTY + 2 * NQ,
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
// One pass over the 128 scores of this thread's row in 32-column chunks.
// KPT: per-thread K groups ((col/64)*8 + col%8) else per-64-key groups.
template <bool KPT>
__device__ __forceinline__ int kgrp(int col) {
  return KPT ? ((col >> 6) << 3) + (col & 7) : (col >> 6);
}

template <bool KPT, bool PV8>
__device__ __forceinline__ void softmax_tile(uint32_t taddr, const float (&c)[16], bool masked, int col0,
                                             int lim, float& m, float& l, float& alpha_out,
                                             uint32_t alpha_bar_full, uint32_t alpha_bar_empty,
                                             uint32_t alpha_parity, float* alpha_slot,
                                             volatile int* abort_flag, uint32_t* err, bool out_bf16,
                                             bool& ok) {
  // pass 1: integer maximum per scale group (c > 0, so max(S*c) = c*max(S))
  int mx[16];
#pragma unroll
  for (int g = 0; g < 16; ++g) mx[g] = INT_MIN;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_ld32(taddr + ch * 32, r);
    tmem_wait_ld(r);
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int col = ch * 32 + u;
      const bool valid = !masked || (col0 + col < lim);
      if (valid) mx[kgrp<KPT>(col)] = max(mx[kgrp<KPT>(col)], (int)r[u]);
    }
  }
  float mt = -INFINITY;
#pragma unroll
  for (int g = 0; g < (KPT ? 16 : 2); ++g)
    if (mx[g] != INT_MIN) mt = fmaxf(mt, c[g] * i2f_exact(mx[g]));
  const float m_new = fmaxf(m, mt);
  const float alpha = (m == -INFINITY) ? 0.f : ex2(m - m_new);
  alpha_out = alpha;
  // publish alpha for the correction warpgroup
  if (!mbar_wait(alpha_bar_empty, alpha_parity ^ 1u, abort_flag, err, kErrTimeoutSoftmax)) { ok = false; return; }
  *alpha_slot = alpha;
  mbar_arrive(alpha_bar_full);

  // pass 2: P~ = 2^(s - m_new) (times 448 in FP8 mode: the static scale is
  // folded into the exponent), row sum, P~ packed over the S columns
  const float bias = PV8 ? (m_new - kLog2Fp8Max) : m_new;
  float lsum = 0.f;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_ld32(taddr + ch * 32, r);
    tmem_wait_ld(r);
    float pv[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int col = ch * 32 + u;
      const float s = fmaf(i2f_exact((int)r[u]), c[kgrp<KPT>(col)], -bias);
      float p = ex2(s);
      if (masked && !(col0 + col < lim)) p = 0.f;
      pv[u] = p;
      lsum += p;
    }
    if (PV8) {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = pack_e4m3x4(pv[4 * k], pv[4 * k + 1], pv[4 * k + 2], pv[4 * k + 3]);
      tmem_st8(taddr + ch * 8, w);
    } else {
      uint32_t w[16];
      if (out_bf16) {
#pragma unroll
        for (int k = 0; k < 16; ++k) w[k] = pack_bf16x2(pv[2 * k], pv[2 * k + 1]);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) w[k] = pack_f16x2(pv[2 * k], pv[2 * k + 1]);
      }
      tmem_st16(taddr + ch * 16, w);
    }
  }
  l = alpha * l + lsum;
  m = m_new;
}

// ---------------------------------------------------------------- kernel
template <int D, bool PV8, bool ACC2>
__global__ void __launch_bounds__(AttnCfg<D, PV8, ACC2>::NTHREADS, 1) attn_fwd_kernel(const AttnParams p) {
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
      auto issue_s = [&](int t) -> bool {
        const int st = t % NST;
        if (!mbar_wait(bar(C::B_KFULL + st), (t / NST) & 1, abort_flag, p.err, kErrTimeoutMma)) return false;
        tc_fence_after();
        for (int q = 0; q < NQ; ++q) {
          if (t >= n[q]) continue;
          const uint32_t d = tmem + C::TM_S + (q * NSB + t % NSB) * 128;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t a = smem_desc(sb + C::OFF_Q + q * C::QT + kk * 32, D);
            const uint64_t bd = smem_desc(sb + C::OFF_K + st * C::QT + kk * 32, D);
            mma_i8_ss(d, a, bd, ID_QK, kk > 0);
          }
          tc_commit(bar(C::B_SFULL + q * NSB + t % NSB));
        }
        tc_commit(bar(C::B_KEMPTY + st));
        return true;
      };
      for (int t = 0; t < NSB && t < maxn && ok; ++t) ok = issue_s(t);
      for (int j = 0; j < maxn && ok; ++j) {
        const int st = j % NST;
        if (!(ok = mbar_wait(bar(C::B_VFULL + st), (j / NST) & 1, abort_flag, p.err, kErrTimeoutMma))) break;
        tc_fence_after();
        for (int q = 0; q < NQ && ok; ++q) {
          if (j >= n[q]) continue;
          ok = mbar_wait(bar(C::B_PFULL + q), j & 1, abort_flag, p.err, kErrTimeoutMma);
          if (ok && (!ACC2 || j > 0))
            ok = mbar_wait(bar(C::B_OREADY + q), (ACC2 ? (j - 1) : j) & 1, abort_flag, p.err, kErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = tmem + C::TM_S + (q * NSB + j % NSB) * 128;
          const uint32_t d = tmem + C::TM_O + q * D;
          if (PV8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = smem_desc(sb + C::OFF_V + st * C::VT + kk * 32, 128);
              mma_f8_ts(d, a0 + kk * 8, bd, ID_PV, ACC2 ? (kk > 0) : (j > 0 || kk > 0));
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd =
                  smem_desc(sb + C::OFF_V + st * C::VT + (kk >> 2) * (D * 128) + (kk & 3) * 32, 128);
              mma_f16_ts(d, a0 + kk * 8, bd, ID_PV, ACC2 ? (kk > 0) : (j > 0 || kk > 0));
            }
          }
          tc_commit(bar(C::B_OFULL + q));
        }
        if (!ok) break;
        tc_commit(bar(C::B_VEMPTY + st));
        if (j + NSB < maxn) ok = issue_s(j + NSB);
      }
      // all MMAs issued by this thread complete before teardown
      tc_commit(bar(C::B_DONE));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(C::B_DONE), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
    }
  } else if (warp >= 4 && warp < 4 + 4 * NQ) {
    // ------------------------------------------------------------ softmax
    const int q = (warp - 4) >> 2;
    const int t = tid - 128 * (1 + q);
    const int qt = pair * NQ + q;
    const uint32_t lane_off = (uint32_t)((t & ~31)) << 16;
    float m = -INFINITY, l = 0.f;
    if (n[q] > 0) {
      const float qsc = p.q_scale[((size_t)h * p.tiles_q + tq0 + qt) * kQGroupsMax + q_group(p.gran, t)];
      const float* ksb = p.k_scale + ((size_t)hk * p.tiles_k + tk0) * kKGroupsMax;
      const bool kpt = p.gran == 2;
      const int row = qt * kTile + t;
      for (int j = 0; j < n[q]; ++j) {
        const int buf = j % NSB;
        if (!mbar_wait(bar(C::B_SFULL + q * NSB + buf), (j / NSB) & 1, abort_flag, p.err, kErrTimeoutSoftmax)) break;
        tc_fence_after();
        float c[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) c[g] = (kpt || g < 2) ? (qsc * __ldg(ksb + j * kKGroupsMax + g)) * p.sl2 : 0.f;
        // keys past the sequence, or (causal) past this row, are masked
        const int col0 = j * kTile;
        const bool masked = (col0 + kTile > Lk) || (p.causal && j == qt);
        const int lim = p.causal ? min(Lk, row + 1) : Lk;
        const uint32_t taddr = tmem + C::TM_S + (q * NSB + buf) * 128 + lane_off;
        const int ab = j & 1;
        float alpha;
        bool ok = true;
        if (kpt)
          softmax_tile<true, PV8>(taddr, c, masked, col0, lim, m, l, alpha, bar(C::B_AFULL + 2 * q + ab),
                                  bar(C::B_AEMPTY + 2 * q + ab), (j >> 1) & 1, alpha_s + (q * 2 + ab) * 128 + t,
                                  abort_flag, p.err, p.out_bf16 != 0, ok);
        else
          softmax_tile<false, PV8>(taddr, c, masked, col0, lim, m, l, alpha, bar(C::B_AFULL + 2 * q + ab),
                                   bar(C::B_AEMPTY + 2 * q + ab), (j >> 1) & 1, alpha_s + (q * 2 + ab) * 128 + t,
                                   abort_flag, p.err, p.out_bf16 != 0, ok);
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + q));
      }
    }
    l_s[q * 128 + t] = l;
    mbar_arrive(bar(C::B_LFULL + q));
  } else if (warp >= 4 + 4 * NQ) {
    // ------------------------------------------------------------ correction + epilogue
    const int t = tid - 128 * (1 + NQ);
    const uint32_t lane_off = (uint32_t)((t & ~31)) << 16;
    bool ok = true;
    float oacc[ACC2 ? D : 1];
#pragma unroll
    for (int i = 0; i < (ACC2 ? D : 1); ++i) oacc[i] = 0.f;
    for (int j = 0; j < maxn && ok; ++j) {
      for (int q = 0; q < NQ && ok; ++q) {
        if (j >= n[q]) continue;
        const int ab = j & 1;
        if (!(ok = mbar_wait(bar(C::B_AFULL + 2 * q + ab), (j >> 1) & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
        const float alpha = alpha_s[(q * 2 + ab) * 128 + t];
        mbar_arrive(bar(C::B_AEMPTY + 2 * q + ab));
        const uint32_t ob = tmem + C::TM_O + q * D + lane_off;
        if (ACC2) {
          if (!(ok = mbar_wait(bar(C::B_OFULL + q), j & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t r[16];
            tmem_ld16(ob + ch * 16, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int u = 0; u < 16; ++u) oacc[ch * 16 + u] = fmaf(alpha, oacc[ch * 16 + u], __uint_as_float(r[u]));
          }
        } else if (j > 0) {
          if (!(ok = mbar_wait(bar(C::B_OFULL + q), (j - 1) & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t r[32];
              tmem_ld32(ob + ch * 32, r);
              tmem_wait_ld(r);
#pragma unroll
              for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
              tmem_st32(ob + ch * 32, r);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(bar(C::B_OREADY + q));
      }
    }
    // epilogue: out = O * (delta_V / l)   (FP8: l sums 448 * P~, O sums
    // P8 * V8, so the 448 cancels) or O / l (16-bit)
    const float* vsc = p.v_scale + ((size_t)b * p.Hkv + hk) * D;
    for (int q = 0; q < NQ && ok; ++q) {
      const int qt = pair * NQ + q;
      const int row = qt * kTile + t;
      if (qt * kTile >= Lq) continue;
      float l = 0.f;
      if (n[q] > 0) {
        if (!ACC2 && !(ok = mbar_wait(bar(C::B_OFULL + q), (n[q] - 1) & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
        if (!(ok = mbar_wait(bar(C::B_LFULL + q), 0, abort_flag, p.err, kErrTimeoutCorr))) break;
        tc_fence_after();
        l = l_s[q * 128 + t];
      }
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + (long long)b * p.os.sb + (long long)h * p.os.sh +
                       (long long)(qs + row) * p.os.ss;
      const uint32_t ob = tmem + C::TM_O + q * D + lane_off;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        float o[32];
        if (ACC2) {
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = oacc[ch * 32 + u];
        } else {
          uint32_t r[32];
          if (n[q] > 0) {
            tmem_ld32(ob + ch * 32, r);
            tmem_wait_ld(r);
          }
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = n[q] > 0 ? __uint_as_float(r[u]) : 0.f;
        }
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float a = o[2 * k] * inv_l, bb = o[2 * k + 1] * inv_l;
          if (PV8) {
            a *= __ldg(vsc + ch * 32 + 2 * k);
            bb *= __ldg(vsc + ch * 32 + 2 * k + 1);
          }
          w[k] = p.out_bf16 ? pack_bf16x2(a, bb) : pack_f16x2(a, bb);
        }
        if (row < Lq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
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
