// CUDA-core tile core of the decode kernel: fp32 FMA dot products for any
// storage type (fp32 or bf16), used for fp32 pools and as the bf16 baseline.
//
// One warp processes a 16-token tile of one KV head for its G grouped query
// heads.  Lane (tg, u) owns the 16-byte unit u of each K/V row and the tokens
// tg*R .. tg*R+R-1 of the tile (U units per row, TG = 32/U token groups, R =
// 16/TG tokens per lane, E elements per unit):
//   1. scores: each lane forms the partial dot products of its unit for its R
//      tokens and G heads (q held in registers, pre-scaled by scale*log2 e);
//      a butterfly reduce-scatter over the U lanes of a token group leaves
//      every (token, head) score complete in exactly one lane;
//   2. online softmax ([P3] eq. (4)): scores go through a per-warp shared
//      buffer; lanes are regrouped as (head, token range) to take the tile
//      max, p = 2^(s - m'), the rescale factor 2^(m - m') and the running l;
//      masked slots (at or past the length) score -inf and give p = 0;
//   3. values: each lane accumulates p * V over its R tokens for its unit
//      and all G heads (o in registers); rows past the length are skipped,
//      never multiplied, so stale NaN slots cannot leak in.
// Shared-memory rows are read as whole 128-byte lines by 8 lanes at a time,
// so the unswizzled TMA layout is free of bank conflicts.
#pragma once

#include "pkv_decode_common.cuh"

namespace pkv {

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }
constexpr int round_up(int x, int a) { return (x + a - 1) / a * a; }

template <typename T, int D, int G>
struct FmaCore {
  static constexpr int ESZ = Elem<T>::kBytes;
  static constexpr int ROWB = D * ESZ;  // bytes per token row of one KV head
  static constexpr int U = ROWB / 16;
  static constexpr int LOGU = ilog2(U);
  static constexpr int TG = 32 / U;
  static constexpr int R = kTile / TG;
  static constexpr int E = 16 / ESZ;
  static constexpr int N = G * R;
  static constexpr int LOGN = ilog2(N);
  static constexpr int RSL = LOGU < LOGN ? LOGU : LOGN;  // reduce-scatter levels
  static constexpr int NF = N >> RSL;                    // scores left per lane
  static constexpr int LPH = (32 / G) < 16 ? (32 / G) : 16;  // softmax lanes per head
  static constexpr int TPL = kTile / LPH;                    // tokens per softmax lane
  static constexpr int TILEB = kTile * ROWB;
  static constexpr int QB = G * ROWB;
  static constexpr int kAlign = 128;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = TILEB;
  static constexpr int kQOff = 2 * TILEB;
  static constexpr int kStageBytes = round_up(2 * TILEB + QB, 128);
  static constexpr int kChunks = 1;          // TMA boxes across a row
  static constexpr int kBoxInner = D;        // elements per box row
  static constexpr int kChunkRowBytes = ROWB;
  static constexpr int kChunkBytes = TILEB;
  static constexpr bool kSwizzle = false;
  static constexpr int kBlockRows = kTile;  // boxes of up to 16 rows, [row] layout
  static constexpr int kScratchBytes = round_up((kTile * G + G) * 4, 16);

  static_assert(U >= 8 && U <= 32, "row must be 128, 256 or 512 bytes");
  static_assert(G >= 1 && G <= 16 && (G & (G - 1)) == 0, "group must be a power of two <= 16");

  struct State {
    float q[G][E];
    float o[G][E];
    float m;  // running max of head lane/LPH (log2 domain), softmax lanes
    float l;  // this lane's share of the running sum
  };

  static PKV_DEVINL void load_unit(const char* p, float (&f)[E]) {
    if constexpr (ESZ == 2) {
      const uint4 w = *reinterpret_cast<const uint4*>(p);
      f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
      f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
    } else {
      const float4 w = *reinterpret_cast<const float4*>(p);
      f[0] = w.x; f[1] = w.y; f[2] = w.z; f[3] = w.w;
    }
  }

  // Byte offset of 16-byte unit `unit` of token row t in a K or V tile.
  static PKV_DEVINL uint32_t row_unit(int t, int unit) { return static_cast<uint32_t>(t * ROWB + unit * 16); }

  static PKV_DEVINL void begin_pair(State& st, const char* qsm, float scale_log2, int lane) {
    const int u = lane & (U - 1);
#pragma unroll
    for (int k = 0; k < G; ++k) {
      float f[E];
      load_unit(qsm + k * ROWB + u * 16, f);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        st.q[k][e] = f[e] * scale_log2;
        st.o[k][e] = 0.f;
      }
    }
    st.m = -INFINITY;
    st.l = 0.f;
  }

  template <class Lim>
  static PKV_DEVINL void tile(State& st, const char* ksm, const char* vsm, const Lim& L,
                              float* scratch, int lane) {
    const int nvalid = L.nvalid;
    const int u = lane & (U - 1);
    const int tg = lane >> LOGU;
    float* sbuf = scratch;               // [kTile][G] scores, then p
    float* abuf = scratch + kTile * G;   // [G] rescale factors

    // 1. partial dot products, idx = k * R + r
    float X[N];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float kf[E];
      load_unit(ksm + (tg * R + r) * ROWB + u * 16, kf);
#pragma unroll
      for (int k = 0; k < G; ++k) {
        float acc = st.q[k][0] * kf[0];
#pragma unroll
        for (int e = 1; e < E; ++e) acc = fmaf(st.q[k][e], kf[e], acc);
        X[k * R + r] = acc;
      }
    }
    // butterfly reduce-scatter over the U lanes of the token group
#pragma unroll
    for (int lev = 0; lev < LOGU; ++lev) {
      const int m = U >> (lev + 1);
      if (lev < RSL) {
        const int half = N >> (lev + 1);
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float a = X[i], b = X[i + half];
          const float send = upper ? a : b;
          const float keep = upper ? b : a;
          X[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      } else {
        X[0] += __shfl_xor_sync(0xffffffffu, X[0], m);
      }
    }
    const int hb = u >> (LOGU - RSL);
    const bool owner = (u & ((1 << (LOGU - RSL)) - 1)) == 0;
#pragma unroll
    for (int i = 0; i < NF; ++i) {
      const int idx = hb * NF + i;
      const int k = idx / R, r = idx % R;
      const int t = tg * R + r;
      const float s = t < L.lim(k) ? X[i] : -INFINITY;
      if (owner) sbuf[t * G + k] = s;
    }
    __syncwarp();

    // 2. online softmax, lanes regrouped as (head kh, tokens li*TPL ..)
    const int kh = lane / LPH, li = lane % LPH;
    const bool active = kh < G;
    float sv[TPL];
    float mt = -INFINITY;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      sv[i] = active ? sbuf[(li * TPL + i) * G + kh] : -INFINITY;
      mt = fmaxf(mt, sv[i]);
    }
#pragma unroll
    for (int msk = 1; msk < LPH; msk <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, msk));
    const float m_new = fmaxf(st.m, mt);
    // no valid score yet for this head: subtract 0 so every exponent is 0, not NaN
    float m_ref = m_new;
    if constexpr (Lim::causal) m_ref = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = exp2f(st.m - m_ref);
    float psum = 0.f;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const float p = exp2f(sv[i] - m_ref);
      psum += p;
      if (active) sbuf[(li * TPL + i) * G + kh] = p;
    }
    st.l = st.l * alpha + psum;
    st.m = m_new;
    if (active && li == 0) abuf[kh] = alpha;
    __syncwarp();

    // 3. rescale and accumulate p * V
    float al[G];
    bool rescale = false;
#pragma unroll
    for (int k = 0; k < G; ++k) {
      al[k] = abuf[k];
      rescale |= al[k] != 1.f;
    }
    if (rescale) {
#pragma unroll
      for (int k = 0; k < G; ++k)
#pragma unroll
        for (int e = 0; e < E; ++e) st.o[k][e] *= al[k];
    }
    if (nvalid >= kTile) {
#pragma unroll
      for (int r = 0; r < R; ++r) accumulate_row(st, vsm, sbuf, tg * R + r, u);
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (tg * R + r < nvalid) accumulate_row(st, vsm, sbuf, tg * R + r, u);
    }
    __syncwarp();
  }

  static PKV_DEVINL void accumulate_row(State& st, const char* vsm, const float* sbuf, int t, int u) {
    float vf[E];
    load_unit(vsm + t * ROWB + u * 16, vf);
    float p[G];
    if constexpr (G % 4 == 0) {
#pragma unroll
      for (int k = 0; k < G; k += 4) {
        const float4 w = *reinterpret_cast<const float4*>(sbuf + t * G + k);
        p[k] = w.x; p[k + 1] = w.y; p[k + 2] = w.z; p[k + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < G; ++k) p[k] = sbuf[t * G + k];
    }
#pragma unroll
    for (int k = 0; k < G; ++k)
#pragma unroll
      for (int e = 0; e < E; ++e) st.o[k][e] = fmaf(p[k], vf[e], st.o[k][e]);
  }

  // Reduce the warp's state and write either the final output (complete
  // pair) or a partial state (o[G][D], m[G], l[G]) for the merge kernel.
  static PKV_DEVINL void finish(State& st, bool complete, void* out, int out_dtype,
                                const OutMap& om, float* part, int lane, float* lse = nullptr) {
    const int u = lane & (U - 1);
    const int tg = lane >> LOGU;
#pragma unroll
    for (int msk = U; msk < 32; msk <<= 1)
#pragma unroll
      for (int k = 0; k < G; ++k)
#pragma unroll
        for (int e = 0; e < E; ++e) st.o[k][e] += __shfl_xor_sync(0xffffffffu, st.o[k][e], msk);
    float l = st.l;
#pragma unroll
    for (int msk = 1; msk < LPH; msk <<= 1) l += __shfl_xor_sync(0xffffffffu, l, msk);
    float lk[G], mk[G];
#pragma unroll
    for (int k = 0; k < G; ++k) {
      lk[k] = __shfl_sync(0xffffffffu, l, k * LPH);
      mk[k] = __shfl_sync(0xffffffffu, st.m, k * LPH);
    }
    if (complete) {
      if (lane < G) {
        float ml = mk[0], ll = lk[0];
#pragma unroll
        for (int k = 1; k < G; ++k)
          if (lane == k) ml = mk[k], ll = lk[k];
        om.put_lse(lse, lane, ml, ll);
      }
      if (tg == 0) {
#pragma unroll
        for (int k = 0; k < G; ++k) {
          const float inv = lk[k] > 0.f ? 1.f / lk[k] : 0.f;  // 0: nothing attended
          float v[E];
#pragma unroll
          for (int e = 0; e < E; ++e) v[e] = st.o[k][e] * inv;
          if (k < om.ncols) store_out(out, out_dtype, om.row(k) + size_t(u) * E, v);
        }
      }
    } else {
      if (tg == 0) {
#pragma unroll
        for (int k = 0; k < G; ++k) {
          float* dst = part + k * D + u * E;
#pragma unroll
          for (int e = 0; e < E; e += 4)
            *reinterpret_cast<float4*>(dst + e) =
                make_float4(st.o[k][e], st.o[k][e + 1], st.o[k][e + 2], st.o[k][e + 3]);
        }
      }
      const int kk = lane % G;
      const float my_m = __shfl_sync(0xffffffffu, st.m, kk * LPH);
      const float my_l = __shfl_sync(0xffffffffu, l, kk * LPH);
      if (lane < G) {
        part[G * D + lane] = my_m;
        part[G * D + G + lane] = my_l;
      }
    }
  }

  template <int NE>
  static PKV_DEVINL void store_out(void* out, int out_dtype, size_t off, const float (&v)[NE]) {
    if (out_dtype == 1) {  // PKV_F32
      float* o = reinterpret_cast<float*>(out) + off;
#pragma unroll
      for (int e = 0; e < NE; e += 4)
        *reinterpret_cast<float4*>(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    } else {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + off;
      uint32_t w[NE / 2];
#pragma unroll
      for (int e = 0; e < NE; e += 2) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[e], v[e + 1]);
        w[e / 2] = *reinterpret_cast<uint32_t*>(&h);
      }
      if constexpr (NE == 8) {
        *reinterpret_cast<uint4*>(o) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        *reinterpret_cast<uint2*>(o) = make_uint2(w[0], w[1]);
      }
    }
  }
};

}  // namespace pkv
