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
// B200 design.  A persistent grid, one CTA (384 threads) per SM, walks work
// items of NQ query tiles of 128 rows of one (sequence, head); the mbarrier
// phases and the K/V ring run on from one item to the next, and the next
// item's first QK^T runs during the current item's epilogue:
//   warp 0        loader: one bulk copy per MMA-ready tile (the pre-pass wrote
//                 tiles already in the swizzled operand layout), NST stages;
//   warp 1        MMA issuer: tcgen05.mma kind::i8 (S = Q K^T, SMEM x SMEM ->
//                 TMEM s32) and kind::f8f6f4 / kind::f16 (O += P~ V, SMEM x
//                 SMEM -> TMEM f32);
//   warp 2        tensor-memory allocation;
//   WG 1..NQ      softmax, one thread per query row (TMEM lane).  It loads its
//                 row of S and at once releases the S columns, so the next
//                 tile's QK^T runs while it works; P~ goes to shared memory in
//                 the swizzled K-major operand layout; in one-level mode it
//                 also rescales O in TMEM and writes the epilogue (dense: the
//                 rows staged as output tensor-map boxes and written with
//                 bulk tensor stores);
//   WG 2 (two-level mode, NQ = 1) correction: adds each tile's fresh partial
//                 O (FP32, or binary16 in fp32+fp16 mode) into an FP32
//                 register accumulator; epilogue.
// Warpgroup 0 (loader, MMA, allocator) hands registers to WG 1..2 with
// setmaxnreg (56 / 224 / 224 per thread).  The softmax's template variants
// (per_thread K scales, bf16 P~, smooth Q) sit behind a run-time switch in the
// one-level kernels and get a kernel each in two-level mode (VAR).
// Every mbarrier wait is bounded (sage_common.cuh): a wait that never ends sets
// the device error word and the CTA tears down instead of hanging.
#include "sage_launch.cuh"

namespace sage {

template <int D, bool PV8, bool ACC2>
struct AttnCfg {
  static constexpr int NQ = ACC2 ? 1 : 2;          // query tiles per CTA
  static constexpr int NST = PV8 ? 3 : 2;          // K/V pipeline stages
  static constexpr int NTHREADS = 384;             // 3 warpgroups (168 registers per thread at launch)
  // per-thread registers after the split: loader / MMA warpgroup, compute
  // warpgroups; 128 * (REGS_LOAD + 2 * REGS_COMPUTE) = NTHREADS * REGS_LAUNCH
  static constexpr int REGS_LAUNCH = 168, REGS_LOAD = 56, REGS_COMPUTE = 224;
  static_assert(128 * (REGS_LOAD + 2 * REGS_COMPUTE) == NTHREADS * REGS_LAUNCH, "register split");
  static constexpr int QT = kTile * D;             // bytes of a Q or K tile
  static constexpr int VT = D * kTile * (PV8 ? 1 : 2);
  static constexpr int PT = kTile * kTile * (PV8 ? 1 : 2);   // P~ tile in shared memory
  // P~ buffers per query tile: two in FP8 one-level mode, so that P~_j is
  // written while P~V_{j-1} still reads P~_{j-1} (16-bit tiles do not fit twice)
  static constexpr int NPB = (PV8 && !ACC2) ? 2 : 1;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * QT;
  static constexpr int OFF_V = OFF_K + NST * QT;
  static constexpr int OFF_P = OFF_V + NST * VT;
  static constexpr int OFF_ALPHA = OFF_P + NPB * NQ * PT;     // float [NQ][2][128]   (two-level)
  static constexpr int OFF_L = OFF_ALPHA + NQ * 2 * 128 * 4;  // float [NQ][128]      (two-level)
  static constexpr int OFF_BIAS = OFF_L + NQ * 128 * 4;       // float [NST][NQ][128]  (smooth Q)
  static constexpr int OFF_KSC = OFF_BIAS + NST * NQ * 128 * 4;  // float [NST][16]: each K tile's group scales
  static constexpr int OFF_BAR = OFF_KSC + NST * kKGroupsMax * 4;
  enum {
    B_QFULL = 0,
    B_QEMPTY = B_QFULL + NQ,         // MMA -> loader: the item's last QK^T with this Q tile is done
    B_KFULL = B_QEMPTY + NQ,
    B_KEMPTY = B_KFULL + NST,
    B_VFULL = B_KEMPTY + NST,
    B_VEMPTY = B_VFULL + NST,
    B_SFULL = B_VEMPTY + NST,        // MMA -> softmax: S_j in TMEM
    B_SCONS = B_SFULL + NQ,          // softmax -> MMA: S_j read, its columns are free
    B_PFULL = B_SCONS + NQ,          // softmax -> MMA: P~_j in shared memory (and O rescaled)
    B_OFULL = B_PFULL + NQ,          // MMA -> softmax / correction: PV_j done
    B_OREADY = B_OFULL + NQ,         // correction -> MMA: partial O consumed (two-level)
    B_AFULL = B_OREADY + NQ,         // softmax -> correction: alpha (two-level)
    B_AEMPTY = B_AFULL + 2 * NQ,
    B_LFULL = B_AEMPTY + 2 * NQ,     // softmax -> correction: final row sum (two-level)
    B_LEMPTY = B_LFULL + NQ,         // correction -> softmax: row sum read
    B_DONE = B_LEMPTY + NQ,
    B_TOK = B_DONE + 1,              // FP8: exponential-phase token, [0] query tile 0 may run, [1] tile 1 may
    B_GO = B_TOK + 2,                // 16-bit: softmax 0 -> softmax 1, start after tile 0's maximum
    NBAR = B_GO + 1
  };
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // [0] tmem base, [1] abort flag
  static constexpr int SMEM_USED = OFF_MISC + 16;
  // At least 116 KB so that a single CTA holds an SM: the CTA allocates all
  // 512 TMEM columns, a second resident CTA would only wait for them.
  static constexpr int SMEM_BYTES = (SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024) + 1024;
  static constexpr int TM_S = 0;                   // S[q] at q * 128
  static constexpr int TM_O = NQ * 128;            // O[q] at TM_O + q * D
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

// Phase 1 of a tile for one query row.  Each column of r holds the float
// t = 1.5 * 2^23 + S exactly (|S| < 2^22): the S accumulator was seeded with
// that bit pattern before the MMA added the int32 products (one-level), or
// the pattern was added to the int32 sums in registers (two-level).
// Masked keys -> -inf; returns the tile maximum m_tile = max_g c_g *
// max_g(S) (c > 0 keeps the order; t is monotonic in S).
template <bool KPT>
__device__ __forceinline__ float tile_max(uint32_t (&r)[128], const float (&c)[16], bool masked, int col0, int lim) {
  if (masked) {
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if (!(col0 + i < lim)) r[i] = 0xFF800000u;   // -inf
  }
  auto F = [&](int i) { return __uint_as_float(r[i]); };
  float mt = -INFINITY;
  if (KPT) {
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      const int base = (g >> 3) * 64 + (g & 7);
      float a = max3(F(base), F(base + 8), F(base + 16));
      float bb = max3(F(base + 24), F(base + 32), F(base + 40));
      a = max3(a, bb, fmaxf(F(base + 48), F(base + 56)));
      mt = fmaxf(mt, c[g] * (a - 12582912.0f));
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
      mt = fmaxf(mt, c[g] * (max3(a0, a1, fmaxf(a2, a3)) - 12582912.0f));
    }
  }
  return mt;
}

// Smooth-Q phase 1: the score of key j is s_j = S_j * c_g(j) + b_j * sl2,
// b_j the tile's per-key correction (shared memory, the same for every row).
// Each column of r is rewritten to s_j (float bits; masked keys -inf) and the
// row maximum is returned.
template <bool KPT>
__device__ __forceinline__ float tile_max_bias(uint32_t (&r)[128], const float (&c)[16], const float* bias,
                                               float sl2, bool masked, int col0, int lim) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int k0 = 0; k0 < 128; k0 += 4) {
    const float4 bb = *reinterpret_cast<const float4*>(bias + k0);
    float b0, b1, b2, b3, s0, s1, s2, s3;
    mul2(b0, b1, bb.x, bb.y, sl2, sl2);
    mul2(b2, b3, bb.z, bb.w, sl2, sl2);
    add2(s0, s1, __uint_as_float(r[k0]), __uint_as_float(r[k0 + 1]), -12582912.0f, -12582912.0f);
    add2(s2, s3, __uint_as_float(r[k0 + 2]), __uint_as_float(r[k0 + 3]), -12582912.0f, -12582912.0f);
    fma2(s0, s1, s0, s1, c[kgrp<KPT>(k0)], c[kgrp<KPT>(k0 + 1)], b0, b1);
    fma2(s2, s3, s2, s3, c[kgrp<KPT>(k0 + 2)], c[kgrp<KPT>(k0 + 3)], b2, b3);
    if (masked) {
      if (!(col0 + k0 < lim)) s0 = -INFINITY;
      if (!(col0 + k0 + 1 < lim)) s1 = -INFINITY;
      if (!(col0 + k0 + 2 < lim)) s2 = -INFINITY;
      if (!(col0 + k0 + 3 < lim)) s3 = -INFINITY;
    }
    r[k0] = __float_as_uint(s0);
    r[k0 + 1] = __float_as_uint(s1);
    r[k0 + 2] = __float_as_uint(s2);
    r[k0 + 3] = __float_as_uint(s3);
    m0 = max3(m0, s0, s1);
    m1 = max3(m1, s2, s3);
  }
  return fmaxf(m0, m1);
}

// Phase 2: P~ = 2^(S*c - m) (times 448 in FP8 mode: the static scale is
// folded into the exponent), the row sum, and P~ rounded to E4M3 / 16 bits
// and stored to row `row` of the shared-memory P~ tile (swizzled K-major,
// 128-byte rows: FP8 one block of 128 keys, 16-bit two blocks of 64 keys).
// Returns the row sum of this tile.


template <bool PV8, bool KPT, bool BF16P, bool BIAS>
__device__ __forceinline__ float tile_exp_store(const uint32_t (&r)[128], const float (&c)[16], float nb,
                                                uint32_t p_smem, int row) {
  auto F = [&](int i) { return __uint_as_float(r[i]); };
  float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // independent partial sums
  const uint32_t rbase = p_smem + row * 128;
  const int sw = row & 7;
  if (PV8) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {          // 16 keys = one 16-byte chunk
      uint32_t w[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int k0 = 16 * ch + 4 * q4;
        float a0, a1, a2, a3;
        if (BIAS) {                                   // r holds the scores
          add2(a0, a1, F(k0), F(k0 + 1), nb, nb);
          add2(a2, a3, F(k0 + 2), F(k0 + 3), nb, nb);
        } else {
          add2(a0, a1, F(k0), F(k0 + 1), -12582912.0f, -12582912.0f);        // exact S
          add2(a2, a3, F(k0 + 2), F(k0 + 3), -12582912.0f, -12582912.0f);
          fma2(a0, a1, a0, a1, c[kgrp<KPT>(k0)], c[kgrp<KPT>(k0 + 1)], nb, nb);
          fma2(a2, a3, a2, a3, c[kgrp<KPT>(k0 + 2)], c[kgrp<KPT>(k0 + 3)], nb, nb);
        }
        const float p0 = ex2(a0), p1 = ex2(a1), p2 = ex2(a2), p3 = ex2(a3);
        add2(ls[2 * (q4 & 1)], ls[2 * (q4 & 1) + 1], ls[2 * (q4 & 1)], ls[2 * (q4 & 1) + 1], p0, p1);
        add2(ls[4 + 2 * (q4 & 1)], ls[5 + 2 * (q4 & 1)], ls[4 + 2 * (q4 & 1)], ls[5 + 2 * (q4 & 1)], p2, p3);
        w[q4] = pack_e4m3x4(p0, p1, p2, p3);
      }
      st_shared_v4(rbase + ((ch ^ sw) << 4), w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {         // 8 keys = one 16-byte chunk
      uint32_t w[4];
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2) {
        const int k0 = 8 * ch + 2 * q2;
        float a0, a1;
        if (BIAS) {
          add2(a0, a1, F(k0), F(k0 + 1), nb, nb);
        } else {
          add2(a0, a1, F(k0), F(k0 + 1), -12582912.0f, -12582912.0f);        // exact S
          fma2(a0, a1, a0, a1, c[kgrp<KPT>(k0)], c[kgrp<KPT>(k0 + 1)], nb, nb);
        }
        const float p0 = ex2(a0), p1 = ex2(a1);
        add2(ls[2 * q2], ls[2 * q2 + 1], ls[2 * q2], ls[2 * q2 + 1], p0, p1);
        w[q2] = BF16P ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
      }
      st_shared_v4(rbase + (ch >> 3) * (kTile * 128) + (((ch & 7) ^ sw) << 4), w[0], w[1], w[2], w[3]);
    }
  }
  return ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
}

// Row epilogue: out[c] = O[c] * inv_l (* delta_V[c] in FP8 mode, where l sums
// 448 * P~ and O sums P8 * V8, so the 448 cancels); 16-bit rounding, one row.
template <int D, bool PV8, bool FROM_REGS>
__device__ __forceinline__ void store_row(uint16_t* orow, uint32_t ob, const float* oacc, float inv_l,
                                          const float* vsc, const float* vmu, bool bf16, bool have_o,
                                          bool valid) {
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
        if (vmu) {                                   // smooth V: the channel mean comes back
          a += __ldg(vmu + ch * 32 + 2 * k);
          bb += __ldg(vmu + ch * 32 + 2 * k + 1);
        }
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

// One-level epilogue of one warp's 32 rows (its quarter of the TMEM lanes):
// out = O * 1/l (* delta_V[c] in FP8 mode, + the channel mean with smooth V),
// rounded to 16 bits.  Each thread puts its row in shared memory, in 16-byte
// chunks, laid out as the boxes of the output tensor map: 64 columns x 32
// rows of 128 bytes, chunk c of row r at c ^ (r mod 8) (the 128-byte
// swizzle), columns 0-63 at stage0 and 64-127 at stage1 (4 KB each: the
// warp's own rows of the query tile's two P~ halves, which only this warp
// writes next).  by_map: the caller stores the boxes with bulk tensor stores;
// otherwise the warp writes whole rows here, one store instruction covering
// 512 contiguous bytes of two (D = 128) or four (D = 64) rows.
template <int D, bool PV8>
__device__ __forceinline__ void store_tile(uint16_t* orow0, long long ss, int nvalid, uint32_t stage0, uint32_t stage1,
                                           uint32_t ob, float inv_l, const float* vsc, const float* vmu, bool bf16,
                                           bool have_o, int lane, bool by_map) {
  constexpr int CH = 2 * D / 16;  // 16-byte chunks per row
  constexpr int RPI = 32 / CH;    // rows per warp store instruction
  auto chunk_addr = [&](int r, int k) -> uint32_t {
    return ((k >> 3) ? stage1 : stage0) + r * 128 + (((k & 7) ^ (r & 7)) << 4);
  };
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t r[32];
    if (have_o) {
      tmem_ld32(ob + ch * 32, r);
      tmem_wait_ld(r);
    }
    uint32_t w[16];
#pragma unroll
    for (int u = 0; u < 8; ++u) {                    // four columns
      float a[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) a[e] = (have_o ? __uint_as_float(r[4 * u + e]) : 0.f) * inv_l;
      if (PV8) {
        const float4 sc = __ldg(reinterpret_cast<const float4*>(vsc + ch * 32) + u);
        a[0] *= sc.x; a[1] *= sc.y; a[2] *= sc.z; a[3] *= sc.w;
        if (vmu) {                                   // smooth V: the channel mean comes back
          const float4 mu = __ldg(reinterpret_cast<const float4*>(vmu + ch * 32) + u);
          a[0] += mu.x; a[1] += mu.y; a[2] += mu.z; a[3] += mu.w;
        }
      }
      w[2 * u] = bf16 ? pack_bf16x2(a[0], a[1]) : pack_f16x2(a[0], a[1]);
      w[2 * u + 1] = bf16 ? pack_bf16x2(a[2], a[3]) : pack_f16x2(a[2], a[3]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int k = ch * 4 + kk;
      st_shared_v4(chunk_addr(lane, k), w[4 * kk], w[4 * kk + 1], w[4 * kk + 2], w[4 * kk + 3]);
    }
  }
  if (by_map) return;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 32 / RPI; ++i) {
    const int rr = i * RPI + lane / CH, k = lane % CH;
    const uint4 v = ld_shared_v4(chunk_addr(rr, k));
    if (rr < nvalid) *reinterpret_cast<uint4*>(orow0 + rr * ss + k * 8) = v;
  }
  __syncwarp();
}

// ---------------------------------------------------------------- work items
// A copy of x that the compiler cannot see through, so that values derived
// from it are recomputed instead of kept live.
__device__ __forceinline__ int opaque(int x) {
  int y;
  asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// A work item is NQ consecutive query tiles (a "pair") of one (sequence,
// head).  The grid is persistent, one CTA per SM: CTA c takes items c,
// c + gridDim.x, c + 2 gridDim.x, ...  Every role walks the same list, so all
// mbarrier phases simply continue from one item to the next.  Non-causal
// items run pair-fastest (the CTAs that run at the same time share K/V in L2);
// causal items run longest first.
template <int NQ>
struct Item {
  int b, h, hk, pair, qs, Lq, Lk, tq0, tk0;
  int n[NQ];   // KV tiles of each query tile (0: the query tile is past the sequence)
  int maxn;
};

// false: the item is empty (past its sequence) or fails a check that the
// pre-pass or the host already reported.
template <int NQ>
__device__ __forceinline__ bool decode_item(const AttnParams& p, int idx, Item<NQ>& it) {
  const int nbh = p.Hq * p.nseq;
  int bh;
  if (p.causal) {
    it.pair = p.n_pairs - 1 - idx / nbh;
    bh = idx % nbh;
  } else {
    it.pair = idx % p.n_pairs;
    bh = idx / p.n_pairs;
  }
  it.h = bh % p.Hq;
  it.b = bh / p.Hq;
  int ks;
  p.seqs.q(it.b, it.qs, it.Lq, it.tq0);
  p.seqs.k(it.b, ks, it.Lk, it.tk0);
  if (p.seqs.cu_q && (it.Lq > p.seqs.max_seqlen || it.Lk > p.seqs.max_seqlen || it.Lq < 0 || it.Lk < 0))
    return false;
  if (it.pair * NQ * kTile >= it.Lq) return false;
  it.hk = it.h / p.group;
  const int nk = (it.Lk + kTile - 1) / kTile;
  // the workspace must hold every tile the item reads (varlen: the offsets
  // kernel has already flagged an overflow)
  if (it.tq0 + (it.Lq + kTile - 1) / kTile > p.tiles_q || it.tk0 + nk > p.tiles_k) return false;
  it.maxn = 0;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int qt = it.pair * NQ + q;
    it.n[q] = qt * kTile >= it.Lq ? 0 : (p.causal ? min(nk, qt + 1) : nk);
    it.maxn = max(it.maxn, it.n[q]);
  }
  return true;
}

// KV tiles of query tile q of an item, without indexing the array by a
// run-time q (which would put the item in local memory).
template <int NQ>
__device__ __forceinline__ int item_n(const Item<NQ>& it, int q) {
  return (NQ == 1 || q == 0) ? it.n[0] : it.n[NQ - 1];
}

// The next item after idx in this CTA's list that has KV tiles.
template <int NQ>
__device__ __forceinline__ bool next_busy_item(const AttnParams& p, int idx, Item<NQ>& it) {
  for (idx += gridDim.x; idx < p.n_items; idx += gridDim.x)
    if (decode_item<NQ>(p, idx, it) && it.maxn > 0) return true;
  return false;
}

// One softmax warpgroup: for each item, the online softmax of query tile q
// over its KV tiles; in one-level mode also the O rescale and the epilogue.
template <int D, bool PV8, bool ACC2, bool A16, bool KPT, bool BF16P, bool SMQ>
__device__ __forceinline__ void softmax_role(const AttnParams& p, const CUtensorMap* out_map, uint32_t sb,
                                             uint32_t tmem, int warp, int tid) {
  using C = AttnCfg<D, PV8, ACC2>;
  constexpr int NQ = C::NQ;
  constexpr bool KSC_SMEM = KPT && !ACC2;   // K group scales from shared memory (see the tile loop)
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  uint8_t* smem = reinterpret_cast<uint8_t*>(__cvta_shared_to_generic(sb));
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* alpha_s = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  float* l_s = reinterpret_cast<float*>(smem + C::OFF_L);

  const int q = (warp - 4) >> 2;
  const int t = tid - 128 * (1 + q);
  const uint32_t lane_off = (uint32_t)((t & ~31)) << 16;
  const bool bf16 = BF16P || (PV8 && p.out_bf16 != 0);
  const uint32_t taddr = tmem + C::TM_S + q * 128 + lane_off;
  const uint32_t ob = tmem + C::TM_O + q * D + lane_off;
  bool ok = true;
  // Phases that run on across items, packed into one register (the tile loop
  // is at the register limit): parity of S_j arrivals, of P~ tiles handed to
  // the MMA (= PVs issued) and whether there was one, of FP8 token turns and
  // 16-bit go signals, the two-level alpha slot (mod 4) and l hand-off parity
  // and whether there was one, and the warpgroup of the previous busy item's
  // last exponential phase (FP8 token; 3 = none).
  enum : uint32_t { PH_S = 1, PH_PV = 2, PH_PVANY = 4, PH_TOK = 8, PH_GO = 16, PH_L = 32, PH_LANY = 64,
                    PH_A0 = 128 /* 2 bits */, PH_LAST0 = 512 /* 2 bits */ };
  uint32_t ph = 3u * PH_LAST0;
  int kvbase = 0;       // K/V ring index of the item's first tile

  // one-level: seed the S columns for the first QK^T (see tile_max)
  if (!ACC2) {
    tmem_fill128(taddr, 0x4B400000u);
    tmem_wait_st();
  }
  tc_fence_before();
  mbar_arrive(bar(C::B_SCONS + q));

  for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
    Item<NQ> it;
    if (!decode_item<NQ>(p, idx, it)) continue;
    const int qt = it.pair * NQ + q;
    const int row = qt * kTile + t;
    const int nq = item_n<NQ>(it, q);
    if (!ACC2 && p.use_out_map) {
      // the previous item's output stores have read the staging area that
      // this item's P~ and epilogue overwrite
      if ((t & 31) == 0) bulk_wait_read0();
      __syncwarp();
    }
    // FP8 token: warpgroup of the next busy item's first exponential phase
    int next_first = -1;
    if (PV8 && NQ == 2 && it.maxn > 0) {
      Item<NQ> nx;
      if (next_busy_item<NQ>(p, idx, nx)) next_first = nx.n[0] > 0 ? 0 : 1;
    }
    float m = -INFINITY, l = 0.f;
    if (nq > 0) {
      const float qsc = p.q_scale[((size_t)it.h * p.tiles_q + it.tq0 + qt) * kQGroupsMax + q_group(p.gran, t)];
      // K group scales: one-level per-thread mode reads each tile's 16 from
      // shared memory, where they arrive with the V tile (16 live registers
      // less in the tile loop); the other modes keep the next tile's few
      // scales in registers, fetched one tile ahead (measured faster there)
      const float* ksb = p.k_scale + ((size_t)it.hk * p.tiles_k + it.tk0) * kKGroupsMax;
      float ksn[KSC_SMEM ? 1 : (KPT ? 16 : 2)];
      if constexpr (!KSC_SMEM) {
#pragma unroll
        for (int g = 0; g < (KPT ? 16 : 2); ++g) ksn[g] = __ldg(ksb + g);
      }
      if (!PV8 && NQ == 2 && q == 1 && it.n[0] > 0) {
        if (!(ok = mbar_wait(bar(C::B_GO), (ph / PH_GO) & 1, abort_flag, p.err, kErrTimeoutSoftmax))) break;
      }
      for (int j = 0; j < nq; ++j) {
        const int kv = kvbase + j;
        float c[16];
        if constexpr (KSC_SMEM) {
          // the tile's K group scales (and, smooth Q, its key corrections)
          // arrive with its V tile
          if (!(ok = mbar_wait(bar(C::B_VFULL + kv % C::NST), (kv / C::NST) & 1, abort_flag, p.err,
                               kErrTimeoutSoftmax)))
            break;
          const float* ksc = reinterpret_cast<const float*>(smem + C::OFF_KSC + (kv % C::NST) * (kKGroupsMax * 4));
#pragma unroll
          for (int g = 0; g < 16; ++g) c[g] = fmaxf((qsc * ksc[g]) * p.sl2, 1e-30f);
        } else {
#pragma unroll
          for (int g = 0; g < 16; ++g) c[g] = g < (KPT ? 16 : 2) ? fmaxf((qsc * ksn[g]) * p.sl2, 1e-30f) : 1e-30f;
          if (j + 1 < nq) {
#pragma unroll
            for (int g = 0; g < (KPT ? 16 : 2); ++g) ksn[g] = __ldg(ksb + (j + 1) * kKGroupsMax + g);
          }
        }
        if (!(ok = mbar_wait(bar(C::B_SFULL + q), ph & PH_S, abort_flag, p.err, kErrTimeoutSoftmax))) break;
        ph ^= PH_S;
        tc_fence_after();
        uint32_t r[128];
        tmem_ld128_sync(taddr, r);
        // The S columns are read.  One-level: re-seed them (the stores
        // complete during the max below), then let the next QK^T in -- of
        // this item or the next.  Two-level: S holds the plain int32 sums;
        // adding the seed's bit pattern in registers gives the same float
        // bits t = 1.5 * 2^23 + S (|S| < 2^22), and measured faster there
        // than the tensor-memory stores.
        if (ACC2) {
#pragma unroll
          for (int i = 0; i < 128; ++i) r[i] += 0x4B400000u;
        } else {
          tmem_fill128(taddr, 0x4B400000u);
        }
        // keys past the sequence, or (causal) past this row, are masked
        const int col0 = j * kTile;
        const bool masked = (col0 + kTile > it.Lk) || (p.causal && j == qt);
        const int lim = p.causal ? min(it.Lk, row + 1) : it.Lk;
        float mt;
        if (SMQ) {
          if constexpr (!KSC_SMEM) {
            // the tile's key corrections arrive with its V tile
            if (!(ok = mbar_wait(bar(C::B_VFULL + kv % C::NST), (kv / C::NST) & 1, abort_flag, p.err,
                                 kErrTimeoutSoftmax)))
              break;
          }
          const float* bias =
              reinterpret_cast<const float*>(smem + C::OFF_BIAS + ((kv % C::NST) * NQ + q) * 512);
          mt = tile_max_bias<KPT>(r, c, bias, p.sl2, masked, col0, lim);
        } else {
          mt = tile_max<KPT>(r, c, masked, col0, lim);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::B_SCONS + q));
        // Conditional rescaling: P~ and O stay relative to the reference m,
        // which moves to the running maximum only when this tile's maximum
        // passes m + tau (tau = 0: the plain online softmax).  P~ <= 2^tau, so
        // FP8 P~ takes the static scale 448 * 2^-tau; the epilogue's 1/l, with
        // l summing the scaled P~, divides it out again.
        const bool move = (m == -INFINITY) || (mt > m + (float)p.lazy_tau);
        const float m_new = move ? fmaxf(m, mt) : m;
        const float alpha = (m == -INFINITY) ? 0.f : ex2(m - m_new);
        if (!PV8 && NQ == 2 && q == 0 && j == 0) mbar_arrive(bar(C::B_GO));
        // the PV that last read the P~ buffer must be done before it is
        // rewritten (one buffer; the item's first tile too, since two-level
        // mode has no epilogue wait)
        if (C::NPB == 1 && (ph & PH_PVANY)) {
          if (!(ok = mbar_wait(bar(C::B_OFULL + q), ((ph / PH_PV) & 1) ^ 1, abort_flag, p.err, kErrTimeoutSoftmax)))
            break;
          tc_fence_after();
        }
        const uint32_t p_smem = sb + C::OFF_P + ((j % C::NPB) * NQ + q) * C::PT;
        if (ACC2) {
          const uint32_t a = (ph / PH_A0) & 3;
          const int ab = a & 1;
          if (!(ok = mbar_wait(bar(C::B_AEMPTY + 2 * q + ab), ((a >> 1) & 1) ^ 1, abort_flag, p.err,
                               kErrTimeoutSoftmax)))
            break;
          ph = (ph & ~(3u * PH_A0)) | (((a + 1) & 3) * PH_A0);
          alpha_s[(q * 2 + ab) * 128 + t] = alpha;
          mbar_arrive(bar(C::B_AFULL + 2 * q + ab));
        }
        // FP8 P~ carries the static scale 448 (folded into the exponent); with
        // the binary16 inner accumulation its scale is 1, so that one tile's
        // partial sums (<= 128 * 448) stay inside binary16's range
        const float nb = -((PV8 && !A16) ? (m_new - kLog2Fp8Max + (float)p.lazy_tau) : m_new);
        // FP8 P~V, two query tiles: their exponential phases take turns (tile
        // 0's of KV tile j, then tile 1's, then tile 0's of j+1, ...; over the
        // items of the CTA one after the other), so that each runs at the
        // MUFU's full rate while the other warpgroup does its maximum and O
        // rescale.  A phase waits for the one before it in that order when the
        // other warpgroup ran it, and hands over when the next one is the other's.
        bool give_turn = false;
        if (PV8 && NQ == 2) {
          bool wait_turn;
          const uint32_t prev_last = (ph / PH_LAST0) & 3;
          if (q == 0) {
            wait_turn = j > 0 ? (j - 1 < it.n[1]) : (prev_last == 1);
            give_turn = j < it.n[1] || (j + 1 >= it.n[0] && next_first == 1);
          } else {
            wait_turn = j < it.n[0] || (j == 0 && prev_last == 0);
            give_turn = j + 1 < it.n[0] || (j + 1 >= it.n[1] && next_first == 0);
          }
          if (wait_turn) {
            if (!(ok = mbar_wait(bar(C::B_TOK + q), (ph / PH_TOK) & 1, abort_flag, p.err, kErrTimeoutSoftmax))) break;
            ph ^= PH_TOK;
          }
        }
        const float lt = tile_exp_store<PV8, KPT, BF16P, SMQ>(r, c, nb, p_smem, t);
        if (PV8 && NQ == 2 && give_turn) mbar_arrive(bar(C::B_TOK + (q ^ 1)));
        l = alpha * l + lt;
        m = m_new;
        if (C::NPB == 2 && j > 0) {
          if (!(ok = mbar_wait(bar(C::B_OFULL + q), ((ph / PH_PV) & 1) ^ 1, abort_flag, p.err, kErrTimeoutSoftmax)))
            break;
          tc_fence_after();
        }
        if (!ACC2 && j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O(q) holds the sums of tiles < j
          if (D == 128) {
            uint32_t o[128];
            tmem_ld128_sync(ob, o);
#pragma unroll
            for (int u = 0; u < 128; u += 2) {
              float x0, x1;
              mul2(x0, x1, __uint_as_float(o[u]), __uint_as_float(o[u + 1]), alpha, alpha);
              o[u] = __float_as_uint(x0);
              o[u + 1] = __float_as_uint(x1);
            }
            tmem_st128(ob, o);
          } else {
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t o[32];
              tmem_ld32(ob + ch * 32, o);
              tmem_wait_ld(o);
#pragma unroll
              for (int u = 0; u < 32; u += 2) {
                float x0, x1;
                mul2(x0, x1, __uint_as_float(o[u]), __uint_as_float(o[u + 1]), alpha, alpha);
                o[u] = __float_as_uint(x0);
                o[u + 1] = __float_as_uint(x1);
              }
              tmem_st32(ob + ch * 32, o);
            }
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + q));
        ph = (ph ^ PH_PV) | PH_PVANY;
      }
      if (!ok) break;
    }
    if (!PV8 && NQ == 2 && q == 1 && it.n[0] > 0) ph ^= PH_GO;   // tile 0 signals once per item
    if (!ACC2 && PV8) {
      // this item's V scales (and means) for the epilogue, into L1
      const size_t vo = ((size_t)it.b * p.Hkv + it.hk) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        prefetch_l1(p.v_scale + vo + c);
        if (p.v_mean) prefetch_l1(p.v_mean + vo + c);
      }
    }
    if (!ACC2) {
      // the next item's Q and K scales, into L1 during the epilogue (in
      // two-level mode the extra work in the softmax costs more than it saves)
      Item<NQ> nx;
      if (next_busy_item<NQ>(p, opaque(idx), nx) && item_n<NQ>(nx, q) > 0) {
        prefetch_l1(p.q_scale + ((size_t)nx.h * p.tiles_q + nx.tq0 + nx.pair * NQ + q) * kQGroupsMax + q_group(p.gran, t));
        if (!KSC_SMEM) prefetch_l1(p.k_scale + ((size_t)nx.hk * p.tiles_k + nx.tk0) * kKGroupsMax);
      }
    }
    if (it.maxn > 0) {
      kvbase += it.maxn;
      ph = (ph & ~(3u * PH_LAST0)) | ((it.n[NQ - 1] == it.maxn ? NQ - 1u : 0u) * PH_LAST0);
    }
    if (ACC2) {
      if (nq > 0) {
        // the correction warpgroup has read the previous item's l
        if ((ph & PH_LANY) &&
            !(ok = mbar_wait(bar(C::B_LEMPTY + q), ((ph / PH_L) & 1) ^ 1, abort_flag, p.err, kErrTimeoutSoftmax)))
          break;
        l_s[q * 128 + t] = l;
        mbar_arrive(bar(C::B_LFULL + q));
        ph = (ph ^ PH_L) | PH_LANY;
      }
    } else if (qt * kTile < it.Lq) {
      // epilogue of this query tile; the MMA already runs the next item's
      // first QK^T meanwhile
      if (nq > 0) {
        if (!(ok = mbar_wait(bar(C::B_OFULL + q), ((ph / PH_PV) & 1) ^ 1, abort_flag, p.err, kErrTimeoutSoftmax)))
          break;
        tc_fence_after();
      }
      // the item's output coordinates, recomputed here rather than kept in
      // registers through the tile loop
      Item<NQ> io;
      decode_item<NQ>(p, opaque(idx), io);
      const float* vsc = p.v_scale + ((size_t)io.b * p.Hkv + io.hk) * D;
      const float* vmu = p.v_mean ? p.v_mean + ((size_t)io.b * p.Hkv + io.hk) * D : nullptr;
      const int w = t >> 5, row0 = qt * kTile + 32 * w;
      uint16_t* orow0 = reinterpret_cast<uint16_t*>(p.out) + (long long)io.b * p.os.sb + (long long)io.h * p.os.sh +
                        (long long)(io.qs + row0) * p.os.ss;
      // staging: this warp's rows of the two P~ halves (FP8: the two buffers;
      // 16-bit: the two 64-key halves of the one buffer)
      const uint32_t half = C::NPB == 2 ? (uint32_t)(NQ * C::PT) : (uint32_t)(C::PT / 2);
      const uint32_t stage0 = sb + C::OFF_P + q * C::PT + w * 4096;
      const int nvalid = min(32, max(0, io.Lq - row0));
      const bool by_map = p.use_out_map != 0;
      store_tile<D, PV8>(orow0, p.os.ss, nvalid, stage0, stage0 + half, ob, l > 0.f ? 1.0f / l : 0.f, vsc, vmu, bf16,
                         nq > 0, t & 31, by_map);
      if (by_map) {
        // dense: the boxes go out with asynchronous bulk tensor stores; the
        // staging area is reused only after they have read it (the wait at
        // the next item's start)
        fence_proxy_async_smem();
        __syncwarp();
        if ((t & 31) == 0 && nvalid > 0) {
          tma_store_4d(out_map, stage0, 0, row0, io.h, io.b);
          if (D == 128) tma_store_4d(out_map, stage0 + half, 64, row0, io.h, io.b);
          bulk_commit();
        }
      }
    }
  }
  // no bulk store still reads this CTA's shared memory when it ends
  if (!ACC2 && (t & 31) == 0) bulk_wait_read0();
}

// ---------------------------------------------------------------- kernel
// VAR: the softmax variant, fixed at compile time (0-7: 4 per_thread K
// scales, 2 bf16 P~, 1 smooth-Q correction; the host picks the kernel), or -1
// for all variants behind a run-time switch.  The two-level kernels are built
// per variant: with the eight compiled into one kernel, the smooth-Q ones made
// it spill and the plain per_block path ran 3-4 % slower.  The one-level
// kernels keep the switch, which measured 1-3 % faster for them.
template <int D, bool PV8, bool ACC2, bool A16, int VAR>
__global__ void __launch_bounds__(384, 1) attn_fwd_kernel(const AttnParams p, const __grid_constant__ CUtensorMap out_map) {
  using C = AttnCfg<D, PV8, ACC2>;
  constexpr int NQ = C::NQ, NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* alpha_s = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  float* l_s = reinterpret_cast<float*>(smem + C::OFF_L);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      uint32_t cnt = 1;
      if ((i >= C::B_SCONS && i < C::B_SCONS + NQ) || (i >= C::B_PFULL && i < C::B_PFULL + NQ) ||
          (i >= C::B_OREADY && i < C::B_OREADY + NQ) || (i >= C::B_AFULL && i < C::B_AFULL + 4 * NQ) ||
          (i >= C::B_LFULL && i < C::B_LFULL + 2 * NQ) || i == C::B_TOK || i == C::B_TOK + 1 || i == C::B_GO)
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

  // Register split: the loader / MMA warpgroup gives registers to the two
  // compute warpgroups (softmax, softmax or correction), whose tile loops run
  // at the limit.  There is one release (warpgroup 0, first thing, never
  // waits) and one request per compute warpgroup, and they add up exactly to
  // the launch's 384 x 168 (the host checks that the kernel was built with
  // 168), so every request is met once warpgroup 0 has released.  Nothing
  // gives registers back: the two sides end the CTA separately, through a
  // named barrier, so their register budgets never meet again.
  if (warp < 4) {
    setmaxnreg_dec<C::REGS_LOAD>();
  if (warp == 0) {
    // ------------------------------------------------------------ loader
    // Per item: the Q tiles (once the MMA has finished the previous item's
    // QK^T with them), then K_t, V_t (+ smooth-Q corrections) for every KV
    // tile through the NST-stage ring, whose index runs on across items.
    if (lane == 0) {
      bool ok = true;
      int kv = 0, issued_k = 0, issued_v = 0;
      uint32_t q_loads = 0;   // bit q: parity of Q loads of query tile q so far
      uint32_t q_any = 0;     // bit q: Q tile q was loaded at least once
      for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
        Item<NQ> it;
        if (!decode_item<NQ>(p, idx, it) || it.maxn == 0) continue;
        const int8_t* qb = p.q_codes + ((size_t)it.h * p.tiles_q + it.tq0 + it.pair * NQ) * C::QT;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if (!ok) break;
          if (it.n[q] == 0) continue;
          if (((q_any >> q) & 1) &&
              !(ok = mbar_wait_poll(bar(C::B_QEMPTY + q), ((q_loads >> q) & 1) ^ 1, abort_flag, p.err, kErrTimeoutLoad)))
            break;
          mbar_expect_tx(bar(C::B_QFULL + q), C::QT);
          bulk_g2s(sb + C::OFF_Q + q * C::QT, qb + (size_t)q * C::QT, C::QT, bar(C::B_QFULL + q));
          q_loads ^= 1u << q;
          q_any |= 1u << q;
        }
        if (!ok) break;
        const int8_t* kb = p.k_codes + ((size_t)it.hk * p.tiles_k + it.tk0) * C::QT;
        const uint8_t* vb = p.v_codes + ((size_t)it.hk * p.tiles_k + it.tk0) * (size_t)C::VT;
        const float* ksc_b = p.k_scale + ((size_t)it.hk * p.tiles_k + it.tk0) * kKGroupsMax;
        // smooth Q: bias rows of the valid query tiles (n[q] > 0 for a prefix of q)
        int nbias = 0;
        if (p.q_bias)
#pragma unroll
          for (int q = 0; q < NQ; ++q) nbias += it.n[q] > 0;
        const float* bias_b =
            p.q_bias ? p.q_bias + ((size_t)it.h * p.tiles_q + it.tq0 + it.pair * NQ) * p.bias_ld : nullptr;
        for (int t = 0; t < it.maxn; ++t, ++kv) {
          const int st = kv % NST, u = kv / NST;
          if (u > 0 && !(ok = mbar_wait_poll(bar(C::B_KEMPTY + st), (u - 1) & 1, abort_flag, p.err, kErrTimeoutLoad)))
            break;
          // (debug, host-selected) CTA 0 withholds one K tile: the MMA's wait
          // for it runs out and the CTA aborts -- the test of the timeout path
          if (!(blockIdx.x == 0 && kv == p.dbg_withhold_k)) {
            mbar_expect_tx(bar(C::B_KFULL + st), C::QT);
            bulk_g2s(sb + C::OFF_K + st * C::QT, kb + (size_t)t * C::QT, C::QT, bar(C::B_KFULL + st));
          }
          issued_k = kv + 1;
          if (u > 0 && !(ok = mbar_wait_poll(bar(C::B_VEMPTY + st), (u - 1) & 1, abort_flag, p.err, kErrTimeoutLoad)))
            break;
          mbar_expect_tx(bar(C::B_VFULL + st), C::VT + nbias * 512 + (ACC2 ? 0 : kKGroupsMax * 4));
          bulk_g2s(sb + C::OFF_V + st * C::VT, vb + (size_t)t * C::VT, C::VT, bar(C::B_VFULL + st));
          // one-level: the K tile's group scales ride with its V tile (the
          // per-thread softmax reads them before its P~ of this tile; the
          // stage is released only after that tile's last P~V)
          if (!ACC2)
            bulk_g2s(sb + C::OFF_KSC + st * (kKGroupsMax * 4), ksc_b + (size_t)t * kKGroupsMax, kKGroupsMax * 4,
                     bar(C::B_VFULL + st));
          for (int q = 0; q < nbias; ++q)   // smooth Q: the query tiles' corrections for key tile t
            bulk_g2s(sb + C::OFF_BIAS + (st * NQ + q) * 512, bias_b + (size_t)q * p.bias_ld + (size_t)t * kTile, 512,
                     bar(C::B_VFULL + st));
          issued_v = kv + 1;
        }
      }
      if (*abort_flag) {
        // let copies in flight land before the CTA's shared memory is released
        for (int t = max(0, issued_k - NST); t < issued_k; ++t) {
          if (blockIdx.x == 0 && t == p.dbg_withhold_k) continue;   // never issued
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(C::B_KFULL + t % NST), (t / NST) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
        for (int t = max(0, issued_v - NST); t < issued_v; ++t) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(C::B_VFULL + t % NST), (t / NST) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
        for (int q = 0; q < NQ; ++q)
          if ((q_any >> q) & 1) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::B_QFULL + q), ((q_loads >> q) & 1) ^ 1) &&
                   global_timer_ns() - t0 < kWaitLimitNs) {}
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per KV tile j of an item: for each query tile, once the softmax has read
    // S_j, S_{j+1} = Q K_{j+1}^T; then for each query tile, once P~_j is in
    // shared memory (and, two-level, the last partial O was consumed),
    // O (+)= P~_j V_j.  S_0 of the next item comes right after the item's
    // last PV (one-level) or before it (two-level) and runs during this item's
    // epilogue.
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_i8(128, 128);
      const uint32_t ID_PV = PV8 ? (A16 ? idesc_e4m3_acc16(128, D) : idesc_e4m3(128, D))
                                 : idesc_f16(128, D, p.out_bf16 != 0);
      bool ok = true;
      int kvs = 0, kvp = 0;                  // ring index of the next K tile (QK^T) and V tile (PV)
      uint32_t s_ph = 0, q_ph = 0, p_ph = 0;  // bit q: parity of S_j seeds, Q loads, P~ tiles consumed
      uint32_t pv_any = 0;                    // bit q: a PV of query tile q was issued
      auto mma_s = [&](int q, int st) {
        const uint32_t d = tmem + C::TM_S + q * 128;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t a = smem_desc(sb + C::OFF_Q + q * C::QT + kk * 32, D);
          const uint64_t bd = smem_desc(sb + C::OFF_K + st * C::QT + kk * 32, D);
          // one-level: onto the 1.5 * 2^23 seed; two-level: the first K chunk
          // overwrites S and the softmax adds the seed's bits itself
          mma_i8_ss(d, a, bd, ID_QK, ACC2 ? (kk > 0) : 1);
        }
        tc_commit(bar(C::B_SFULL + q));
      };
      auto mma_pv = [&](int q, int j, int st) {
        const uint32_t d = tmem + C::TM_O + q * D;
        const uint32_t pa = sb + C::OFF_P + ((j % C::NPB) * NQ + q) * C::PT;
        const uint32_t va = sb + C::OFF_V + st * C::VT;
        if (PV8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ss(d, smem_desc(pa + kk * 32, 128), smem_desc(va + kk * 32, 128), ID_PV,
                      ACC2 ? (kk > 0) : (j > 0 || kk > 0));
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ss(d, smem_desc(pa + (kk >> 2) * (kTile * 128) + (kk & 3) * 32, 128),
                       smem_desc(va + (kk >> 2) * (D * 128) + (kk & 3) * 32, 128), ID_PV,
                       ACC2 ? (kk > 0) : (j > 0 || kk > 0));
        }
        tc_commit(bar(C::B_OFULL + q));
      };
      // S_t of item `it` for every query tile that has KV tile t
      auto issue_s = [&](const Item<NQ>& it, int t) -> bool {
        const int st = kvs % NST;
        if (!mbar_wait_poll(bar(C::B_KFULL + st), (kvs / NST) & 1, abort_flag, p.err, kErrTimeoutMma)) return false;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if (t >= it.n[q]) continue;
          if (t == 0) {
            if (!mbar_wait_poll(bar(C::B_QFULL + q), (q_ph >> q) & 1, abort_flag, p.err, kErrTimeoutMma)) return false;
            q_ph ^= 1u << q;
          }
          if (!mbar_wait_poll(bar(C::B_SCONS + q), (s_ph >> q) & 1, abort_flag, p.err, kErrTimeoutMma)) return false;
          s_ph ^= 1u << q;
          tc_fence_after();
          mma_s(q, st);
          if (t == it.n[q] - 1) tc_commit(bar(C::B_QEMPTY + q));   // the Q tile may be replaced
        }
        tc_commit(bar(C::B_KEMPTY + st));
        ++kvs;
        return true;
      };
      bool s0_issued = false;
      for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
        Item<NQ> it;
        if (!decode_item<NQ>(p, idx, it) || it.maxn == 0) continue;
        if (!s0_issued && !(ok = issue_s(it, 0))) break;
        s0_issued = false;
        for (int j = 0; j < it.maxn; ++j) {
          if (j + 1 < it.maxn) {
            if (!(ok = issue_s(it, j + 1))) break;
          } else if (ACC2) {
            // two-level: the last PV waits for the correction warpgroup, so
            // the next item's first QK^T goes ahead of it
            Item<NQ> nx;
            if (next_busy_item<NQ>(p, idx, nx)) {
              if (!(ok = issue_s(nx, 0))) break;
              s0_issued = true;
            }
          }
          const int st = kvp % NST;
          if (!(ok = mbar_wait_poll(bar(C::B_VFULL + st), (kvp / NST) & 1, abort_flag, p.err, kErrTimeoutMma))) break;
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            if (!ok) break;
            if (j >= it.n[q]) continue;
            ok = mbar_wait_poll(bar(C::B_PFULL + q), (p_ph >> q) & 1, abort_flag, p.err, kErrTimeoutMma);
            if (ok && ACC2 && ((pv_any >> q) & 1))
              ok = mbar_wait_poll(bar(C::B_OREADY + q), ((p_ph >> q) & 1) ^ 1, abort_flag, p.err, kErrTimeoutMma);
            if (!ok) break;
            p_ph ^= 1u << q;
            pv_any |= 1u << q;
            tc_fence_after();
            mma_pv(q, j, st);
          }
          if (!ok) break;
          tc_commit(bar(C::B_VEMPTY + st));
          ++kvp;
          if (!ACC2 && j + 1 == it.maxn) {
            // one-level: the next item's first QK^T after this item's last PV
            // (which need not wait for the next Q tile); it runs during the
            // epilogue
            Item<NQ> nx;
            if (next_busy_item<NQ>(p, idx, nx)) {
              if (!(ok = issue_s(nx, 0))) break;
              s0_issued = true;
            }
          }
        }
      }
      // all MMAs issued by this thread complete before teardown
      tc_commit(bar(C::B_DONE));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(C::B_DONE), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
    }
  }
    __syncwarp();
    tc_fence_before();
    named_bar_sync(1, C::NTHREADS);          // every role has finished
    if (warp == 2) {
      tc_fence_after();
      tmem_dealloc(tmem, C::TM_COLS);
    }
  } else {
    setmaxnreg_inc<C::REGS_COMPUTE>();
  if (warp < 4 + 4 * NQ) {
    // ------------------------------------------------------------ softmax
    const bool bf16p = !PV8 && p.out_bf16;
    const int variant = (p.gran == 2 ? 4 : 0) + (bf16p ? 2 : 0) + (p.q_bias ? 1 : 0);
#define SAGE_SOFTMAX(KPT, BF16P, SMQ) softmax_role<D, PV8, ACC2, A16, KPT, BF16P, SMQ>(p, &out_map, sb, tmem, warp, tid)
    if constexpr (VAR >= 0) {
      (void)variant;
      SAGE_SOFTMAX((VAR & 4) != 0, (VAR & 2) != 0, (VAR & 1) != 0);
    } else {
      switch (variant) {
        case 0: SAGE_SOFTMAX(false, false, false); break;
        case 1: SAGE_SOFTMAX(false, false, true); break;
        case 2: SAGE_SOFTMAX(false, true, false); break;
        case 3: SAGE_SOFTMAX(false, true, true); break;
        case 4: SAGE_SOFTMAX(true, false, false); break;
        case 5: SAGE_SOFTMAX(true, false, true); break;
        case 6: SAGE_SOFTMAX(true, true, false); break;
        default: SAGE_SOFTMAX(true, true, true); break;
      }
    }
#undef SAGE_SOFTMAX
  } else if (ACC2) {
    // ------------------------------------------------------------ correction (two-level) + epilogue
    const int t = tid - 128 * (1 + NQ);
    const uint32_t lane_off = (uint32_t)((t & ~31)) << 16;
    const uint32_t ob = tmem + C::TM_O + lane_off;
    bool ok = true;
    int a_cnt = 0;
    uint32_t o_ph = 0, l_ph = 0;
    for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
      Item<NQ> it;
      if (!decode_item<NQ>(p, idx, it)) continue;
      if (PV8) {
        // the item's V scales (and means) for the epilogue, into L1
        const size_t vo = ((size_t)it.b * p.Hkv + it.hk) * D;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          prefetch_l1(p.v_scale + vo + c);
          if (p.v_mean) prefetch_l1(p.v_mean + vo + c);
        }
      }
      float oacc[D];
#pragma unroll
      for (int i = 0; i < D; ++i) oacc[i] = 0.f;
      for (int j = 0; j < it.n[0]; ++j) {
        const int ab = a_cnt & 1;
        if (!(ok = mbar_wait(bar(C::B_AFULL + ab), (a_cnt >> 1) & 1, abort_flag, p.err, kErrTimeoutCorr))) break;
        ++a_cnt;
        const float alpha = alpha_s[ab * 128 + t];
        mbar_arrive(bar(C::B_AEMPTY + ab));
        if (!(ok = mbar_wait(bar(C::B_OFULL), o_ph, abort_flag, p.err, kErrTimeoutCorr))) break;
        o_ph ^= 1;
        tc_fence_after();
        if (A16) {
          // binary16 partial sums, one per TMEM column; the load packs two
          // adjacent columns into one register
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t r[16];
            tmem_ld32_pack16(ob + ch * 32, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float2 f = h16x2_to_f32x2(r[u]);
              fma2(oacc[ch * 32 + 2 * u], oacc[ch * 32 + 2 * u + 1], alpha, alpha, oacc[ch * 32 + 2 * u],
                   oacc[ch * 32 + 2 * u + 1], f.x, f.y);
            }
          }
        } else {
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
        }
        tc_fence_before();
        mbar_arrive(bar(C::B_OREADY));
      }
      if (!ok) break;
      const int row = it.pair * kTile + t;
      float l = 0.f;
      if (it.n[0] > 0) {
        if (!(ok = mbar_wait(bar(C::B_LFULL), l_ph, abort_flag, p.err, kErrTimeoutCorr))) break;
        l_ph ^= 1;
        l = l_s[t];
        mbar_arrive(bar(C::B_LEMPTY));
      }
      const float* vsc = p.v_scale + ((size_t)it.b * p.Hkv + it.hk) * D;
      const float* vmu = p.v_mean ? p.v_mean + ((size_t)it.b * p.Hkv + it.hk) * D : nullptr;
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + (long long)it.b * p.os.sb + (long long)it.h * p.os.sh +
                       (long long)(it.qs + row) * p.os.ss;
      store_row<D, PV8, true>(orow, ob, oacc, l > 0.f ? 1.0f / l : 0.f, vsc, vmu, p.out_bf16 != 0, true,
                              row < it.Lq);
    }
  }

    __syncwarp();
    tc_fence_before();
    named_bar_sync(1, C::NTHREADS);
  }
  (void)alpha_s;
  (void)l_s;
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
    if (mbar_wait_poll(smem_u32(&bars[0]), 0, &abort_flag, err, kErrTimeoutMma)) {
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
// Persistent grid: one CTA per SM (each holds all of an SM's tensor memory),
// fewer when there are fewer items, or p.max_ctas when that is set (a debug
// cap: results do not depend on the grid).
template <int D, bool PV8, bool ACC2, bool A16, int VAR>
static cudaError_t launch_attn(const AttnParams& p, const CUtensorMap& out_map, cudaStream_t s) {
  using C = AttnCfg<D, PV8, ACC2>;
  auto k = attn_fwd_kernel<D, PV8, ACC2, A16, VAR>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // the register split needs the launch allocation it was sized for: with
  // fewer registers a warpgroup's setmaxnreg.inc would wait for ever
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, k)) != cudaSuccess) return e;
  if (fa.numRegs != C::REGS_LAUNCH) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if (p.max_ctas > 0 && p.max_ctas < sms) sms = p.max_ctas;
  const int grid = p.n_items < sms ? p.n_items : sms;
  k<<<grid, C::NTHREADS, C::SMEM_BYTES, s>>>(p, out_map);
  return cudaGetLastError();
}

// Query tiles per CTA for a configuration (the host sizes the grid with it).
int attn_tiles_per_cta(int D, bool pv8, bool acc2) {
  (void)D; (void)pv8;
  return acc2 ? 1 : 2;
}

// Two-level kernels: the instantiation of softmax variant `var` (the same
// bits as the kernel's run-time switch); bf16 P~ exists only for 16-bit P~V.
template <int D, bool PV8, bool A16, int V = 0>
static cudaError_t launch_two_level(const AttnParams& p, const CUtensorMap& out_map, int var, cudaStream_t s) {
  if constexpr (V > 7) {
    return cudaErrorInvalidValue;
  } else if constexpr (PV8 && (V & 2)) {
    return launch_two_level<D, PV8, A16, V + 1>(p, out_map, var, s);
  } else {
    if (var == V) return launch_attn<D, PV8, true, A16, V>(p, out_map, s);
    return launch_two_level<D, PV8, A16, V + 1>(p, out_map, var, s);
  }
}

template <int D>
static cudaError_t launch_mode(const AttnParams& p, const CUtensorMap& out_map, bool pv8, int acc, cudaStream_t s) {
  const int var = (p.gran == 2 ? 4 : 0) + (!pv8 && p.out_bf16 ? 2 : 0) + (p.q_bias ? 1 : 0);
  if (pv8) {
    if (acc == kAccTwoF16) return launch_two_level<D, true, true>(p, out_map, var, s);
    if (acc == kAccTwo) return launch_two_level<D, true, false>(p, out_map, var, s);
    return launch_attn<D, true, false, false, -1>(p, out_map, s);
  }
  if (acc == kAccTwo) return launch_two_level<D, false, false>(p, out_map, var, s);
  return launch_attn<D, false, false, false, -1>(p, out_map, s);
}

cudaError_t attn_forward(const AttnParams& p0, const CUtensorMap& out_map, int D, bool pv8, int acc, int max_len_q,
                         int nseq, cudaStream_t s) {
  const bool acc2 = acc != kAccOne;
  const int per = attn_tiles_per_cta(D, pv8, acc2) * kTile;
  const long long nx = (max_len_q + per - 1) / per;
  const long long items = nx * p0.Hq * nseq;
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (acc == kAccTwoF16 && !pv8) return cudaErrorInvalidValue;
  AttnParams p = p0;
  p.n_pairs = (int)nx;
  p.nseq = nseq;
  p.n_items = (int)items;
  if (D == 128) return launch_mode<128>(p, out_map, pv8, acc, s);
  return launch_mode<64>(p, out_map, pv8, acc, s);
}

cudaError_t debug_qk_tile(const int8_t* qt, const int8_t* kt, int D, int32_t* out, uint32_t* err,
                          cudaStream_t s) {
  qk_tile_kernel<<<1, 128, 0, s>>>(qt, kt, D, out, err);
  return cudaGetLastError();
}

}  // namespace sage
