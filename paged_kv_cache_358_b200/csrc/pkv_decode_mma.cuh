// Tensor-core tile core of the decode kernel for bf16 pools (mma.sync
// m16n8k16, bf16 inputs, fp32 accumulation).
//
// Decode attention is a streaming read with G flops per byte (G = grouped
// query heads per KV head), far below any tensor-core ridge; the tensor cores
// here only take the multiply-adds off the CUDA cores, whose issue slots
// would otherwise bound the kernel below HBM speed at G = 4..8.  tcgen05 needs
// M >= 64 and a TMEM round trip per tile for the softmax; the warp-level
// m16n8k16 shape fits one 16-token tile and the grouped heads directly.
//
// Shapes per 16-token tile (tokens in M, up to 8 grouped columns in N):
//   scores  S^T[16 tok x 8 cols] = K[16 x D] * Q^T[D x 8]      (D/16 MMAs)
//   values  O^T[D x 8 cols]     += V^T[D x 16 tok] * P^T[16 x 8] (D/16 MMAs)
// (16 columns use MmaCoreM16 below, with the columns in M.)
// K and V tiles arrive through TMA with the 128-byte swizzle, so ldmatrix
// (plain for K, .trans for V^T) reads them without bank conflicts.  The
// score accumulator (token-major) is turned into the P^T operand of the value
// MMA with movmatrix.trans, after the online-softmax update of [P3] eq. (4)
// in fp32 on the accumulator registers.  P is rounded to bf16 for the value
// MMA (relative error <= 2^-9 per weight) while the running sum l adds the
// fp32 weights, so the output's scale is off by at most 2^-9; everything
// else stays fp32.
// Slots at or past the length: their scores are replaced by -inf, and in the
// last tile their V^T operand columns are zeroed before the MMA, so stale NaN
// rows cannot reach the accumulator through 0 * NaN.
#pragma once

#include "pkv_decode_fma.cuh"

namespace pkv {

PKV_DEVINL void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

PKV_DEVINL void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

PKV_DEVINL void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

PKV_DEVINL uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

PKV_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// SB: rows of one block per TMA box.  kTile (block size >= 16, or 8 through
// one box per 128-byte part and block): a tile holds each 128-byte part of
// its 16 rows together, [part][row].  4 (block size 4): one box per block
// brings all parts of its 4 rows, so a tile is [block][part][row]; each box
// still starts on a 1 KiB boundary (head_dim >= 128), as the 128-byte
// swizzle's pattern needs.
template <int D, int G, int SB = kTile>
struct MmaCore {
  static constexpr int ESZ = 2;
  static constexpr int ROWB = D * ESZ;
  static constexpr int NCH = ROWB / 128;      // 128-byte swizzle atoms per row
  static constexpr int KSTEPS = D / 16;
  static constexpr int CHUNKB = kTile * 128;  // one swizzled chunk of a tile
  static constexpr int TILEB = NCH * CHUNKB;
  static constexpr int QB = G * ROWB;
  static constexpr int kAlign = 1024;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = TILEB;
  static constexpr int kQOff = 2 * TILEB;
  static constexpr int kStageBytes = round_up(2 * TILEB + QB, 1024);
  static constexpr int kChunks = NCH;
  static constexpr int kBoxInner = 64;  // bf16 elements per 128-byte box row
  static constexpr int kChunkRowBytes = 128;
  static constexpr int kChunkBytes = CHUNKB;
  static constexpr bool kSwizzle = true;
  static constexpr int kScratchBytes = 0;

  static_assert(G >= 1 && G <= 8, "grouped heads must fit the 8 MMA columns");
  static_assert(NCH >= 1 && NCH <= 4, "head_dim 64, 128 or 256");

  struct State {
    uint32_t qb[KSTEPS][2];  // Q^T B-fragments (bf16x2), heads >= G are zero
    float oc[KSTEPS][4];     // O^T accumulator: rows d = 16*mt + gid (+8), cols heads 2*tig (+1)
    float m[2];              // running max of heads 2*tig, 2*tig+1 (log2 domain)
    float l[2];              // this lane's share of the running sums
  };

  // Byte offset of (row t, 16-byte unit) inside a swizzled tile.
  static constexpr int kBlockRows = SB;  // rows per box when a tile spans several blocks
  static_assert(SB == kTile || (SB == 4 && NCH >= 2), "4-row boxes start on 1 KiB boundaries only with >= 2 parts");

  static PKV_DEVINL uint32_t swz(int t, int unit) {
    if constexpr (SB == kTile) {
      return static_cast<uint32_t>((unit >> 3) * CHUNKB + t * 128 + (((unit & 7) ^ (t & 7)) << 4));
    } else {
      // row r of block b, part p: the swizzle pattern follows the row's
      // position in the 1 KiB-aligned box, p * SB + r
      const int b = t / SB, r = t % SB, p = unit >> 3;
      return static_cast<uint32_t>(b * (SB * ROWB) + p * (SB * 128) + r * 128 +
                                   (((unit & 7) ^ ((p * SB + r) & 7)) << 4));
    }
  }

  // Byte offset of 16-byte unit `unit` of token row t in a K or V tile.
  static PKV_DEVINL uint32_t row_unit(int t, int unit) { return swz(t, unit); }

  static PKV_DEVINL void begin_pair(State& st, const char* qsm, float /*scale_log2*/, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      if (gid < G) {
        const char* row = qsm + gid * ROWB + (16 * kk + 2 * tig) * 2;
        st.qb[kk][0] = *reinterpret_cast<const uint32_t*>(row);
        st.qb[kk][1] = *reinterpret_cast<const uint32_t*>(row + 16);
      } else {
        st.qb[kk][0] = 0u;
        st.qb[kk][1] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) st.oc[kk][i] = 0.f;
    }
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
  }

  template <class Lim>
  static PKV_DEVINL void tile(State& st, const char* ksm, const char* vsm, const Lim& L,
                              float scale_log2, int lane) {
    const int nvalid = L.nvalid;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t kbase = smem_u32(ksm), vbase = smem_u32(vsm);

    // scores S^T = K Q^T, the k-steps alternating between two accumulators so
    // the dependent MMA chain is half as long
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    {
      float c2[4] = {0.f, 0.f, 0.f, 0.f};
      const int t = lane & 15;
      const int cb = lane >> 4;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kbase + swz(t, 2 * kk + cb), a0, a1, a2, a3);
        mma_bf16_16816((kk & 1) ? c2 : c, a0, a1, a2, a3, st.qb[kk][0], st.qb[kk][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) c[i] += c2[i];
    }
    // c[0]: (tok gid, col 2tig), c[1]: (gid, 2tig+1), c[2]: (gid+8, 2tig), c[3]: (gid+8, 2tig+1)
    const int lim0 = L.lim(2 * tig), lim1 = L.lim(2 * tig + 1);
    float s[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = gid + ((i & 2) ? 8 : 0);
      s[i] = t < ((i & 1) ? lim1 : lim0) ? c[i] * scale_log2 : -INFINITY;
    }
    float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
    for (int msk = 4; msk < 32; msk <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, msk));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, msk));
    }
    const float mn0 = fmaxf(st.m[0], mx0), mn1 = fmaxf(st.m[1], mx1);
    // Under the causal mask a column may have seen no valid score yet and keep
    // m = -inf: subtract 0 instead, so every exponent is exp2(-inf) = 0 and
    // nothing becomes NaN.  Without it every tile has a valid row.
    float r0 = mn0, r1 = mn1;
    if constexpr (Lim::causal) {
      r0 = mn0 == -INFINITY ? 0.f : mn0;
      r1 = mn1 == -INFINITY ? 0.f : mn1;
    }
    const float al0 = fast_exp2(st.m[0] - r0), al1 = fast_exp2(st.m[1] - r1);
    st.m[0] = mn0;
    st.m[1] = mn1;
    const float p0 = fast_exp2(s[0] - r0), p1 = fast_exp2(s[1] - r1);
    const float p2 = fast_exp2(s[2] - r0), p3 = fast_exp2(s[3] - r1);
    st.l[0] = st.l[0] * al0 + (p0 + p2);
    st.l[1] = st.l[1] * al1 + (p1 + p3);
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        st.oc[mt][0] *= al0;
        st.oc[mt][1] *= al1;
        st.oc[mt][2] *= al0;
        st.oc[mt][3] *= al1;
      }
    }
    // P^T operand: transpose the token-major fragments
    const uint32_t b0 = movmatrix_trans(pack_bf16x2(p0, p1));
    const uint32_t b1 = movmatrix_trans(pack_bf16x2(p2, p3));

    // values O^T += V^T P^T
    const int vt = ((lane >> 4) << 3) + (lane & 7);
    const int vu = (lane >> 3) & 1;
    uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
    const bool tail = nvalid < kTile;
    if (tail) {
      mlo = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
      mhi = (2 * tig + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 9 < nvalid ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(vbase + swz(vt, 2 * mt + vu), a0, a1, a2, a3);
      if (tail) {
        a0 &= mlo;
        a1 &= mlo;
        a2 &= mhi;
        a3 &= mhi;
      }
      mma_bf16_16816(st.oc[mt], a0, a1, a2, a3, b0, b1);
    }
  }

  static PKV_DEVINL void finish(State& st, bool complete, void* out, int out_dtype, const OutMap& om,
                                float* part, int lane, float* lse = nullptr) {
    const int gid = lane >> 2, tig = lane & 3;
    float l0 = st.l[0], l1 = st.l[1];
#pragma unroll
    for (int msk = 4; msk < 32; msk <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, msk);
      l1 += __shfl_xor_sync(0xffffffffu, l1, msk);
    }
    const int h0 = 2 * tig, h1 = 2 * tig + 1;
    if (complete) {
      const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;  // 0: nothing attended
      if (gid == 0) {
        om.put_lse(lse, h0, st.m[0], l0);
        om.put_lse(lse, h1, st.m[1], l1);
      }
      const size_t r0 = om.row(h0), r1 = om.row(h1);
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        const int d0 = 16 * mt + gid, d1 = d0 + 8;
        if (h0 < om.ncols) {
          put(out, out_dtype, r0 + d0, st.oc[mt][0] * i0);
          put(out, out_dtype, r0 + d1, st.oc[mt][2] * i0);
        }
        if (h1 < om.ncols) {
          put(out, out_dtype, r1 + d0, st.oc[mt][1] * i1);
          put(out, out_dtype, r1 + d1, st.oc[mt][3] * i1);
        }
      }
    } else {
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        const int d0 = 16 * mt + gid, d1 = d0 + 8;
        if (h0 < G) {
          part[h0 * D + d0] = st.oc[mt][0];
          part[h0 * D + d1] = st.oc[mt][2];
        }
        if (h1 < G) {
          part[h1 * D + d0] = st.oc[mt][1];
          part[h1 * D + d1] = st.oc[mt][3];
        }
      }
      if (gid == 0) {
        if (h0 < G) {
          part[G * D + h0] = st.m[0];
          part[G * D + G + h0] = l0;
        }
        if (h1 < G) {
          part[G * D + h1] = st.m[1];
          part[G * D + G + h1] = l1;
        }
      }
    }
  }

  static PKV_DEVINL void put(void* out, int out_dtype, size_t off, float v) {
    if (out_dtype == 1)
      reinterpret_cast<float*>(out)[off] = v;
    else
      reinterpret_cast<__nv_bfloat16*>(out)[off] = __float2bfloat16_rn(v);
  }
};

// Tensor-core core for 16 grouped columns (G = 16, or T query tokens x Gq
// heads = 16), with the columns in the MMA's M dimension:
//   scores  S[16 cols x 16 tok] = Q[16 x D] * K^T[D x 16]   (2 * D/16 MMAs)
//   values  O[16 cols x D]     += P[16 x 16 tok] * V[16 tok x D] (D/8 MMAs)
// The score accumulators of the two 8-token halves are, packed to bf16,
// exactly the A operand of the value product (no transpose), and a column's
// 16 scores sit in the 4 lanes of one quad (2 shuffle levels for its max and
// sum).  K is read with ldmatrix as the B operand, V with ldmatrix.trans.
// Same shared-memory stage layout as MmaCore (TMA 128-byte swizzle).
template <int D, int SB = kTile>
struct MmaCoreM16 {
  using Base = MmaCore<D, 8, SB>;  // tile layout, swizzle and output helpers (independent of G)
  static constexpr int kBlockRows = SB;
  static constexpr int G = 16;
  static constexpr int ESZ = Base::ESZ;
  static constexpr int ROWB = Base::ROWB;
  static constexpr int KSTEPS = D / 16;
  static constexpr int NT = D / 8;  // 8-wide output column tiles
  static constexpr int QB = G * ROWB;
  static constexpr int kAlign = Base::kAlign;
  static constexpr int kKOff = Base::kKOff;
  static constexpr int kVOff = Base::kVOff;
  static constexpr int kQOff = Base::kQOff;
  static constexpr int kStageBytes = round_up(2 * Base::TILEB + QB, 1024);
  static constexpr int kChunks = Base::kChunks;
  static constexpr int kBoxInner = Base::kBoxInner;
  static constexpr int kChunkRowBytes = Base::kChunkRowBytes;
  static constexpr int kChunkBytes = Base::kChunkBytes;
  static constexpr bool kSwizzle = true;
  static constexpr int kScratchBytes = 0;
  static_assert(D <= 128, "the 16-row accumulator of head_dim 256 does not fit the registers");

  struct State {
    uint32_t qa[KSTEPS][4];  // Q A-fragments: rows gid / gid+8, k = 2tig(+1) / 2tig+8(+9)
    float o[NT][4];          // O rows gid / gid+8, cols 8*nt + 2tig (+1)
    float m[2];              // running max of rows gid, gid+8 (log2 domain; equal over a quad)
    float l[2];              // this lane's share of the running sums
  };

  static PKV_DEVINL uint32_t swz(int t, int unit) { return Base::swz(t, unit); }
  static PKV_DEVINL uint32_t row_unit(int t, int unit) { return Base::swz(t, unit); }

  static PKV_DEVINL void begin_pair(State& st, const char* qsm, float /*scale_log2*/, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const char* r0 = qsm + gid * ROWB + (16 * kk + 2 * tig) * 2;
      const char* r1 = r0 + 8 * ROWB;
      st.qa[kk][0] = *reinterpret_cast<const uint32_t*>(r0);
      st.qa[kk][1] = *reinterpret_cast<const uint32_t*>(r1);
      st.qa[kk][2] = *reinterpret_cast<const uint32_t*>(r0 + 16);
      st.qa[kk][3] = *reinterpret_cast<const uint32_t*>(r1 + 16);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) st.o[nt][0] = st.o[nt][1] = st.o[nt][2] = st.o[nt][3] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
  }

  template <class Lim>
  static PKV_DEVINL void tile(State& st, const char* ksm, const char* vsm, const Lim& L, float scale_log2,
                              int lane) {
    const int nvalid = L.nvalid;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t kbase = smem_u32(ksm), vbase = smem_u32(vsm);

    // scores: s0 for tokens 0..7, s1 for tokens 8..15 (C rows = columns)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      // matrices: (tok 0-7, unit 2kk), (tok 0-7, 2kk+1), (tok 8-15, 2kk), (tok 8-15, 2kk+1)
      const int t = (lane & 7) + ((lane >> 4) << 3);
      const int hu = (lane >> 3) & 1;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + swz(t, 2 * kk + hu), b0, b1, b2, b3);
        mma_bf16_16816(s0, st.qa[kk][0], st.qa[kk][1], st.qa[kk][2], st.qa[kk][3], b0, b1);
        mma_bf16_16816(s1, st.qa[kk][0], st.qa[kk][1], st.qa[kk][2], st.qa[kk][3], b2, b3);
      }
    }
    // row gid: s0[0], s0[1], s1[0], s1[1] (tokens 2tig, 2tig+1, 8+2tig, 9+2tig); row gid+8: [2], [3]
    const int lim0 = L.lim(gid), lim1 = L.lim(gid + 8);
    const int t0 = 2 * tig;
    float x[8];
    x[0] = t0 < lim0 ? s0[0] * scale_log2 : -INFINITY;
    x[1] = t0 + 1 < lim0 ? s0[1] * scale_log2 : -INFINITY;
    x[2] = t0 + 8 < lim0 ? s1[0] * scale_log2 : -INFINITY;
    x[3] = t0 + 9 < lim0 ? s1[1] * scale_log2 : -INFINITY;
    x[4] = t0 < lim1 ? s0[2] * scale_log2 : -INFINITY;
    x[5] = t0 + 1 < lim1 ? s0[3] * scale_log2 : -INFINITY;
    x[6] = t0 + 8 < lim1 ? s1[2] * scale_log2 : -INFINITY;
    x[7] = t0 + 9 < lim1 ? s1[3] * scale_log2 : -INFINITY;
    float mx0 = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    float mx1 = fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7]));
#pragma unroll
    for (int msk = 1; msk < 4; msk <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, msk));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, msk));
    }
    const float mn0 = fmaxf(st.m[0], mx0), mn1 = fmaxf(st.m[1], mx1);
    float r0 = mn0, r1 = mn1;
    if constexpr (Lim::causal) {  // a column with no valid score yet: subtract 0, not -inf
      r0 = mn0 == -INFINITY ? 0.f : mn0;
      r1 = mn1 == -INFINITY ? 0.f : mn1;
    }
    const float al0 = fast_exp2(st.m[0] - r0), al1 = fast_exp2(st.m[1] - r1);
    st.m[0] = mn0;
    st.m[1] = mn1;
    float p[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      p[i] = fast_exp2(x[i] - r0);
      p[4 + i] = fast_exp2(x[4 + i] - r1);
    }
    st.l[0] = st.l[0] * al0 + ((p[0] + p[1]) + (p[2] + p[3]));
    st.l[1] = st.l[1] * al1 + ((p[4] + p[5]) + (p[6] + p[7]));
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        st.o[nt][0] *= al0;
        st.o[nt][1] *= al0;
        st.o[nt][2] *= al1;
        st.o[nt][3] *= al1;
      }
    }
    // P as the A operand: rows gid / gid+8, tokens 2tig(+1) and 8+2tig(+1)
    const uint32_t pa0 = pack_bf16x2(p[0], p[1]);
    const uint32_t pa1 = pack_bf16x2(p[4], p[5]);
    const uint32_t pa2 = pack_bf16x2(p[2], p[3]);
    const uint32_t pa3 = pack_bf16x2(p[6], p[7]);

    // values: V as the B operand via ldmatrix.trans; matrices (tok 0-7, unit
    // 2mt), (tok 8-15, 2mt), (tok 0-7, 2mt+1), (tok 8-15, 2mt+1)
    const int vt = (lane & 7) + (((lane >> 3) & 1) << 3);
    const int vu = lane >> 4;
    uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
    const bool tail = nvalid < kTile;
    if (tail) {  // V rows at or past the length never reach the accumulator (0 * NaN)
      mlo = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
      mhi = (2 * tig + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 9 < nvalid ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(vbase + swz(vt, 2 * mt + vu), b0, b1, b2, b3);
      if (tail) {
        b0 &= mlo;
        b1 &= mhi;
        b2 &= mlo;
        b3 &= mhi;
      }
      mma_bf16_16816(st.o[2 * mt], pa0, pa1, pa2, pa3, b0, b1);
      mma_bf16_16816(st.o[2 * mt + 1], pa0, pa1, pa2, pa3, b2, b3);
    }
  }

  static PKV_DEVINL void finish(State& st, bool complete, void* out, int out_dtype, const OutMap& om,
                                float* part, int lane, float* lse = nullptr) {
    const int gid = lane >> 2, tig = lane & 3;
    float l0 = st.l[0], l1 = st.l[1];
#pragma unroll
    for (int msk = 1; msk < 4; msk <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, msk);
      l1 += __shfl_xor_sync(0xffffffffu, l1, msk);
    }
    const int c0 = gid, c1 = gid + 8;
    if (complete) {
      const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;  // 0: nothing attended
      if (tig == 0) {
        om.put_lse(lse, c0, st.m[0], l0);
        om.put_lse(lse, c1, st.m[1], l1);
      }
      const size_t r0 = om.row(c0), r1 = om.row(c1);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int d = 8 * nt + 2 * tig;
        if (c0 < om.ncols) {
          Base::put(out, out_dtype, r0 + d, st.o[nt][0] * i0);
          Base::put(out, out_dtype, r0 + d + 1, st.o[nt][1] * i0);
        }
        if (c1 < om.ncols) {
          Base::put(out, out_dtype, r1 + d, st.o[nt][2] * i1);
          Base::put(out, out_dtype, r1 + d + 1, st.o[nt][3] * i1);
        }
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int d = 8 * nt + 2 * tig;
        *reinterpret_cast<float2*>(part + c0 * D + d) = make_float2(st.o[nt][0], st.o[nt][1]);
        *reinterpret_cast<float2*>(part + c1 * D + d) = make_float2(st.o[nt][2], st.o[nt][3]);
      }
      if (tig == 0) {
        part[G * D + c0] = st.m[0];
        part[G * D + c1] = st.m[1];
        part[G * D + G + c0] = l0;
        part[G * D + G + c1] = l1;
      }
    }
  }
};

}  // namespace pkv
