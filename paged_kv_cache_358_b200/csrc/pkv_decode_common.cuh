// Shared pieces of the decode-attention kernels: workspace layout, the work
// decomposition and the tile-core interface the FMA and MMA cores implement.
//
// The method is PagedAttention decode as "PagedAttention：让 KV cache 按需生长"
// (hs-black.github.io) states it in section
// "分页以后，attention 仍然按完整历史归一化": for each logical block look up the
// physical block, load its K/V tile, mask slots at or past the length, score
// q K^T * scale and apply the online-softmax update; equation (4) of
// "内存预算约束下的语言模型服务：注意力、分页与调度" gives the update
//   m' = max(m, max_j s_j),  l' = e^{m-m'} l + sum_j e^{s_j-m'},
// with the value accumulator rescaled by e^{m-m'}.  Scores are kept in the
// log2 domain (q is pre-multiplied by scale * log2(e)), so every e^x becomes
// 2^x on the same exponent: the same function, one multiply fewer per score.
//
// Work decomposition (our design, not the pages'): a "pair" is (request s,
// KV-head group hg) and its history is cut into 16-token tiles.  All tiles of
// all pairs form one flattened sequence ordered (s, hg, tile), split into
// equal contiguous ranges, one per CTA of a persistent grid (a stream-K over
// CTAs), so every CTA streams the same number of tiles whatever the length
// mix.  Warp w of a CTA takes KV head hg*HG + w of each tile in the range; the
// library runs one-warp CTAs (HG = 1, eight per SM), the width that measured
// fastest.  Each warp runs its own ring of shared-memory stages fed by TMA and
// keeps one (m, l, o) state per grouped query head; when the CTA's range
// covers a whole pair the warp writes the final output, otherwise a partial
// state, and the last CTA to finish a split (request, KV head) merges the
// partial states.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int kTile = 16;          // tokens per tile
constexpr int kMaxBoxes = 4;       // TMA boxes per tile (block_size >= 4)
constexpr int kBatch = 32;         // tiles of block-table lookahead per warp

struct WsHeader {
  uint32_t status;
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t kv_dtype;
  int32_t num_workers;     // CTAs of the partition grid
  int32_t head_groups;     // KV-head groups per request
  int32_t planned;
  int32_t pad;
  long long total_tiles;   // flattened (request, head group, tile) units
};

// Partial state of one (CTA, pair, head-in-group): o[G][D], m[G], l[G],
// padded so every slot starts on a 16-byte boundary.
constexpr int part_stride(int G, int D) { return G * D + ((2 * G + 3) & ~3); }

// Workspace layout (byte offsets, each 256-aligned):
//   header | prefix int32[S+1] (tiles per request, cumulative) |
//   worker plan int4[2*NW] {tile_begin, tile_end, s, offset in s}, {len(s), 0, 0, 0} |
//   arrival counters int32[S*H_kv] (pieces of a split (request, KV head) counted in: low 16
//     bits those that ended their CTA's range, high 16 bits the one flushed mid-range) |
//   partial states float[(NW + S*NHG) * HG][part_stride(G, D)]
struct WsLayout {
  size_t prefix = 0, wplan = 0, counters = 0, partials = 0, total = 0;
  WsLayout() = default;
  static size_t up(size_t x) { return (x + 255) & ~size_t(255); }
  WsLayout(int S, int H_kv, int HG, int G, int D, int NW) {
    const int NHG = H_kv / HG;
    prefix = up(sizeof(WsHeader));
    wplan = prefix + up(sizeof(int32_t) * (size_t(S) + 1));
    counters = wplan + up(2 * sizeof(int4) * size_t(NW));
    partials = counters + up(sizeof(int32_t) * size_t(S) * H_kv);
    total = partials +
            up(sizeof(float) * (size_t(NW) + size_t(S) * NHG) * size_t(HG) * part_stride(G, D));
  }
};

struct DecodeArgs {
  const void* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  void* out;
  char* ws;
  size_t off_prefix, off_wplan, off_counters, off_partials;
  int32_t max_blocks;   // table row stride
  int32_t num_seqs, num_q_heads, num_kv_heads;
  int32_t head_groups;  // NHG = num_kv_heads / HG
  int32_t block_size, num_blocks;
  int32_t out_dtype;
  int32_t num_workers;
  int32_t num_q_tokens;  // T query tokens per request (1 for plain decode)
  int32_t causal;        // T > 1: 1 = token i sees positions < len - (T-1-i); 0 = all see all
  float scale_log2;     // scale * log2(e)
  // Optional log-sum-exp output (null: none): lse[s][i][h] = log2 of the
  // softmax denominator in the log2 domain of the scores (-inf when nothing
  // was attended), for combining this result with another over other tokens.
  float* lse;
  // Folded append (all null when the new tokens were appended separately):
  // row s of k_new / v_new is request s's new token, the last of its history,
  // written to pool slot new_slots[s] (< 0: no new token for s).
  const void* k_new;
  const void* v_new;
  const int64_t* new_slots;
  void* k_pool;
  void* v_pool;
  // 1: launched as a dependent of the plan kernel that writes this launch's
  // plan: wait for it before reading anything (the launch's own start-up
  // then overlaps the plan kernel instead of following it)
  int32_t wait_first;
  // 1: the caller merges the split pieces of a launch whose pairs a later
  // launch merges (merged_by_later_launch) itself: no merge launch behind
  // the partition kernel
  int32_t merge_by_caller;
};

PKV_DEVINL void store1(void* out, int out_dtype, size_t off, float v) {
  if (out_dtype == 1)
    reinterpret_cast<float*>(out)[off] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(out)[off] = __float2bfloat16_rn(v);
}

PKV_DEVINL int ntiles_of(int len) { return len > 0 ? (len + kTile - 1) / kTile : 0; }

// Whether the pools are read through a 5-D tensor map whose box holds every
// 128-byte part of its rows (swizzled rows of more than one part): one box
// per 16-row tile (block size >= 16), or one per block when the tile core
// lays a tile out block by block (block_rows: its rows per block box, 4);
// otherwise a 4-D map, one box per part and block.
__host__ __device__ __forceinline__ bool tile_map_5d(int row_bytes, int part_bytes, int box_rows, bool swizzle,
                                                     int block_rows) {
  return swizzle && row_bytes > part_bytes && (box_rows == kTile || box_rows == block_rows);
}

// Worker that owns flattened tile t when T tiles are split over NW workers
// (worker v owns [floor(v T / NW), floor((v+1) T / NW))).
PKV_DEVINL int owner_of(long long t, long long T, int NW) {
  return static_cast<int>(((t + 1) * NW - 1) / T);
}
PKV_DEVINL long long range_begin(int v, long long T, int NW) {
  return (static_cast<long long>(v) * T) / NW;
}

// Valid rows of a tile for each column of the grouped computation.  A column
// is (query token i, grouped head k), c = i * Gq + k.  With T query tokens per
// request at the last T positions, token i sees positions < len - (T-1-i)
// (causal); rows at or past the length hold no data at all.  Single-token
// decode (kCausal = false) masks by the length alone, with no per-column work.
template <bool kCausal>
struct TileLim {
  static constexpr bool causal = kCausal;  // columns may differ, and may see no row
  int nvalid;  // rows holding tokens of the request (1..16)
  int rem;     // length - first position of the tile (may exceed 16)
  int T;       // query tokens per request
  int gq_mul;  // ceil(2^16 / Gq): c / Gq == (c * gq_mul) >> 16 for every column c < 16
  int causal_on;  // 0: the T tokens all see the whole history (columns differ only in q)
  PKV_DEVINL int lim(int c) const {
    if constexpr (!kCausal) {
      return nvalid;
    } else {
      if (!causal_on) return nvalid;
      const int causal_lim = rem - (T - 1 - ((c * gq_mul) >> 16));
      return causal_lim < nvalid ? causal_lim : nvalid;
    }
  }
};

// Output row of column c: out[s][i][head * Gq + k][:] for c = i * Gq + k,
// given the row of column 0 and the stride between query tokens (H_q * d).
// Columns c >= ncols (= T * Gq, padded up to the kernel's power-of-two group)
// are not written.
struct OutMap {
  size_t row0;
  size_t tok_stride;
  int Gq;
  int D;
  int ncols;
  PKV_DEVINL size_t row(int c) const {
    if (ncols == Gq) return row0 + static_cast<size_t>(c) * D;  // one token: rows are adjacent
    return row0 + static_cast<size_t>(c / Gq) * tok_stride + static_cast<size_t>(c % Gq) * D;
  }
  // Optional log-sum-exp output (lse null: none), one value per output row:
  // log2 of the softmax denominator of column c from its running max m and sum l.
  PKV_DEVINL void put_lse(float* lse, int c, float m, float l) const {
    if (lse != nullptr && c < ncols) lse[row(c) / static_cast<size_t>(D)] = l > 0.f ? m + __log2f(l) : -INFINITY;
  }
};

// Per-stage metadata written by the issuing lane, read by the consuming warp.
struct alignas(16) StageMeta {
  int32_t s;       // request
  int32_t hg;      // head group
  int32_t j;       // tile index within the pair
  int32_t flags;   // bit 0: first tile of a pair in this warp (q staged); bit 1: the pair's last
                   // tile; bits 8..: valid tokens in the tile
  int32_t nt;      // tiles of the pair
  int32_t new_slot;  // folded append: pool slot of the pair's new token (< 0: none)
  int32_t len;       // length of the request
  int32_t pad;
};

}  // namespace pkv
