// Partition-kernel templates of the decode attention and the host-side
// launch helpers that instantiate them.  Included by one translation unit per
// (storage type, head_dim) so the variants compile in parallel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/pkv.h"
#include <type_traits>

#include "pkv_decode_mma.cuh"
#include "pkv_host.h"

namespace pkv {

// ---------------------------------------------------------------------------
// Merge of a split (request, KV head), run by one warp of the last CTA to
// finish it: combine the partial states (m_u, l_u, o_u) of CTAs u = v0..v1 with
//   M = max_u m_u,  l = sum_u 2^(m_u - M) l_u,  o = sum_u 2^(m_u - M) o_u,
// and write o / l -- the online-softmax rescaling rule applied to states.
// Lanes read the (CTA, head) states of a pass together, so the merge costs a
// couple of memory round trips, not one per CTA.
// ---------------------------------------------------------------------------
// The log-sum-exp output of a general (MULTI) launch, for the merge: passing
// it as one more argument would change the register allocation of the
// streaming loop around the call.
__shared__ float* s_lse_out;

// Kept out of line: its load batches need many registers for a moment, and
// inlined they would raise the register count of the whole streaming loop.
template <int D, int G, int HG, bool MULTI>
__device__ __noinline__ void merge_pair(const float* partials, long long pp, int w, int v0, int v1, long long T,
                           int NW, void* out, int out_dtype, OutMap om, int lane) {
  constexpr int PS = part_stride(G, D);
  constexpr int PER = D / 32;   // output elements per lane
  constexpr int UMAX = 32 / G;  // CTAs per pass: lane i reads (CTA i / G, head i % G)
  constexpr int NE = UMAX * G;  // (CTA, head) entries per pass (32)
  constexpr int CH = 16;        // entries whose o slices are loaded per round trip
  auto slot = [&](int u) { return partials + (static_cast<size_t>(u + pp) * HG + w) * PS; };
  const int kk = lane % G;
  float run_m = -INFINITY;  // running max of query head kk (replicated over lanes with equal kk)
  float run_l = 0.f;        // running sum of query head kk
  float acc[G][PER];
#pragma unroll
  for (int k = 0; k < G; ++k)
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[k][i] = 0.f;
  for (int u0 = v0; u0 <= v1; u0 += UMAX) {
    // Every load reads a written slot: CTAs past v1 or without tiles are
    // replaced by v0 (which always holds a state) and weighted 0, so no load
    // waits behind a data-dependent branch.  The m/l loads and the first
    // chunk of o loads go out together.
    const int uu = u0 + lane / G;
    const bool valid = uu <= v1 && (T >= NW || range_begin(uu, T, NW) < range_begin(uu + 1, T, NW));
    const int my_slot = valid ? uu : v0;  // entry `lane` of this pass
    const float* su = slot(my_slot);
    float mv = __ldcg(su + G * D + kk);
    const float lv = __ldcg(su + G * D + G + kk);
    float vals[CH][PER];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const float* src = slot(__shfl_sync(0xffffffffu, my_slot, c)) + (c % G) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) vals[c][i] = __ldcg(src + i);
    }
    if (!valid) mv = -INFINITY;
    float mk = mv;
#pragma unroll
    for (int msk = G; msk < 32; msk <<= 1) mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, msk));
    const float nm = fmaxf(run_m, mk);
    // under the causal mask a column no CTA saw a token for keeps m = -inf:
    // subtract 0 there, not -inf
    const float nms = (MULTI && nm == -INFINITY) ? 0.f : nm;
    const float old_scale = exp2f(run_m - nms);  // 0 on the first pass
    const float wgt = valid ? exp2f(mv - nms) : 0.f;
    float wl = wgt * lv;
#pragma unroll
    for (int msk = G; msk < 32; msk <<= 1) wl += __shfl_xor_sync(0xffffffffu, wl, msk);
    run_l = run_l * old_scale + wl;
    run_m = nm;
#pragma unroll
    for (int k = 0; k < G; ++k) {
      const float sk = __shfl_sync(0xffffffffu, old_scale, k);
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[k][i] *= sk;
    }
#pragma unroll
    for (int j0 = 0; j0 < NE; j0 += CH) {
      if (j0 > 0) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int j = j0 + c;
          const float* src = slot(__shfl_sync(0xffffffffu, my_slot, j)) + (j % G) * D + lane * PER;
#pragma unroll
          for (int i = 0; i < PER; ++i) vals[c][i] = __ldcg(src + i);
        }
      }
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int j = j0 + c;
        const float wj = __shfl_sync(0xffffffffu, wgt, j);  // 0 for replaced entries
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[j % G][i] = fmaf(wj, vals[c][i], acc[j % G][i]);
      }
    }
  }
  if constexpr (MULTI) {  // lane k holds column k's running max and sum
    if (lane < G) om.put_lse(s_lse_out, lane, run_m, run_l);
  }
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const float lk = __shfl_sync(0xffffffffu, run_l, k);
    if constexpr (MULTI) {
      const float inv = lk > 0.f ? 1.f / lk : 0.f;  // a column with no visible token is 0
      if (k < om.ncols)
#pragma unroll
        for (int i = 0; i < PER; ++i) store1(out, out_dtype, om.row(k) + lane * PER + i, acc[k][i] * inv);
    } else {
      const float inv = 1.f / lk;
#pragma unroll
      for (int i = 0; i < PER; ++i) store1(out, out_dtype, om.row0 + k * D + lane * PER + i, acc[k][i] * inv);
    }
  }
}

// Which workers hold the pieces of the split pair (request s, KV head `head`),
// from the plan alone (its header, the request's length and tile offset):
// nothing the partition kernel writes, so a merge may find its span before it
// waits for that kernel.  Returns false when there is nothing to merge (the
// pair was not split, the request is empty, or the plan is for another shape
// -- which the partition kernel recorded).
struct MergeSpan {
  long long pp;  // pair index s * NHG + head
  long long TT;  // tiles of the launch
  int v0, v1;    // first and last worker holding a piece
  int NW;
};
__device__ __forceinline__ bool merge_span(const DecodeArgs& a, int check_Hq, int check_dtype, int D, int s,
                                           int head, MergeSpan& m) {
  const int NW = a.num_workers, NHG = a.head_groups;
  // one round trip: the plan's header, the request's length and tile offset
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(a.ws + a.off_prefix);
  const int planned = __ldcg(&hdr->planned), h_s = __ldcg(&hdr->num_seqs), h_hq = __ldcg(&hdr->num_q_heads);
  const int h_hkv = __ldcg(&hdr->num_kv_heads), h_d = __ldcg(&hdr->head_dim), h_dt = __ldcg(&hdr->kv_dtype);
  const int h_nw = __ldcg(&hdr->num_workers), h_nhg = __ldcg(&hdr->head_groups);
  const long long TT = __ldcg(&hdr->total_tiles);
  const int len = __ldcg(a.seq_lens + s);
  const int pre = __ldcg(prefix + s);
  if (planned != 1 || h_s != a.num_seqs || h_hq != check_Hq || h_hkv != a.num_kv_heads || h_d != D ||
      h_dt != check_dtype || h_nw != NW || h_nhg != NHG)
    return false;
  const int nt = ntiles_of(len);
  if (nt == 0) return false;  // zeros, written by the partition kernel
  // one-warp workers: the head group is the KV head
  const long long pstart = static_cast<long long>(pre) * NHG + static_cast<long long>(head) * nt;
  if (pstart < 0 || pstart + nt > TT) return false;  // lengths changed since the plan (recorded there)
  m.v0 = owner_of(pstart, TT, NW);
  m.v1 = owner_of(pstart + nt - 1, TT, NW);
  if (m.v0 == m.v1) return false;  // the whole pair was in one CTA, which wrote it
  m.pp = static_cast<long long>(s) * NHG + head;
  m.TT = TT;
  m.NW = NW;
  return true;
}

// Merge of column c of a split pair from its pieces, as the partition kernel
// left them in the workspace `a.ws` (call after waiting for that kernel): M
// (the max, log2 domain), L (the sum) and the lane's D/32 output elements,
// not yet divided by L.  One round trip loads every piece's m and l and the o
// slices of the first UB pieces together (the o loads need no weight); more
// than UB pieces take one more round trip per UB.
template <int D, int G, bool MULTI>
__device__ __forceinline__ void merge_pieces(const DecodeArgs& a, const MergeSpan& m, int c, int lane, float& M,
                                             float& L, float (&acc)[D / 32]) {
  constexpr int PS = part_stride(G, D);
  constexpr int PER = D / 32;  // output elements per lane
  constexpr int UB = 8;        // pieces whose o slices are loaded together
  const int v0 = m.v0, v1 = m.v1;
  const float* partials = reinterpret_cast<const float*>(a.ws + a.off_partials);
  // workers are one-warp CTAs (head group 1, which launch_core requires), so
  // worker u's piece of the pair is slot u + pp
  auto slot = [&](int u) { return partials + static_cast<size_t>(u + m.pp) * PS; };
  // CTAs without tiles (fewer tiles than workers) hold no state
  auto valid = [&](int u) { return m.TT >= m.NW || range_begin(u, m.TT, m.NW) < range_begin(u + 1, m.TT, m.NW); };
  // UB o slices in flight.  Pieces past the batch, and CTAs without tiles
  // (their slots were never written and may hold any bits, NaN included),
  // read piece v0 instead, which always holds a state, with weight 0.
  auto load_batch = [&](float (&vals)[UB][PER], int first, int nb) {
#pragma unroll
    for (int j = 0; j < UB; ++j) {
      const int uj = (j < nb && valid(first + j)) ? first + j : v0;
      const float* src = slot(uj) + c * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; i += 4 <= PER ? 4 : PER) {
        if constexpr (PER >= 4) {
          const float4 f = __ldcg(reinterpret_cast<const float4*>(src + i));
          vals[j][i] = f.x; vals[j][i + 1] = f.y; vals[j][i + 2] = f.z; vals[j][i + 3] = f.w;
        } else {
          const float2 f = __ldcg(reinterpret_cast<const float2*>(src + i));
          vals[j][i] = f.x; vals[j][i + 1] = f.y;
        }
      }
    }
  };
  // the pieces' maxima and sums: lane j holds pieces v0 + j, v0 + j + 32, ...
  // (up to 32 pieces in registers, the common case; more are re-read)
  float mj = -INFINITY, lj = 0.f;
  if (v0 + lane <= v1 && valid(v0 + lane)) {
    mj = __ldcg(slot(v0 + lane) + G * D + c);
    lj = __ldcg(slot(v0 + lane) + G * D + G + c);
  }
  const int nb0 = v1 - v0 + 1 < UB ? v1 - v0 + 1 : UB;
  float vals[UB][PER];
  load_batch(vals, v0, nb0);
  M = mj;
  for (int u = v0 + 32 + lane; u <= v1; u += 32)
    if (valid(u)) M = fmaxf(M, __ldcg(slot(u) + G * D + c));
#pragma unroll
  for (int msk = 16; msk > 0; msk >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, msk));
  // under the causal mask a column no piece saw a token for keeps M = -inf:
  // subtract 0 there, so every weight is 0
  const float Ms = (MULTI && M == -INFINITY) ? 0.f : M;
  L = exp2f(mj - Ms) * lj;
  for (int u = v0 + 32 + lane; u <= v1; u += 32)
    if (valid(u)) L += exp2f(__ldcg(slot(u) + G * D + c) - Ms) * __ldcg(slot(u) + G * D + G + c);
#pragma unroll
  for (int msk = 16; msk > 0; msk >>= 1) L += __shfl_xor_sync(0xffffffffu, L, msk);
  const float w0 = exp2f(mj - Ms);  // 0 for an empty or missing piece (mj = -inf)
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  auto accumulate = [&](const float (&vals)[UB][PER], float w, int j0, int nb) {
#pragma unroll
    for (int j = 0; j < UB; ++j) {
      const float wj = __shfl_sync(0xffffffffu, w, (j0 + j) & 31);
      const float ww = j0 + j < nb ? wj : 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(ww, vals[j][i], acc[i]);
    }
  };
  accumulate(vals, w0, 0, nb0);
  // pieces past the first batch (more than UB of them: rare)
  for (int u0 = v0; u0 <= v1; u0 += 32) {
    const int u = u0 + lane;
    float w = w0;
    if (u0 != v0) w = (u <= v1 && valid(u)) ? exp2f(__ldcg(slot(u) + G * D + c) - Ms) : 0.f;
    const int nb = v1 - u0 + 1 < 32 ? v1 - u0 + 1 : 32;
    for (int j0 = (u0 == v0 ? UB : 0); j0 < nb; j0 += UB) {
      load_batch(vals, u0 + j0, nb - j0);
      accumulate(vals, w, j0, nb);
    }
  }
}

// ---------------------------------------------------------------------------
// Merge of the split pairs of a 16-column launch, as a kernel of its own
// launched right behind the partition kernel (a programmatic dependent
// launch).  With 16 columns a pair's partial states are 8 KB per piece, and
// one warp merging ~6 of them needs about nine dependent L2 round trips
// (about 30,000 cycles, measured), run at the very end of the launch by one
// CTA per pair while every other SM idles.  Here one warp per (pair, column)
// merges its column over the whole GPU: its pair's span from the plan before
// waiting for the partition kernel (merge_span), then one round trip for the
// pieces' m and l and o slices together (merge_pieces).  Same rule as
// merge_pair:
//   M = max_u m_u,  l = sum_u 2^(m_u - M) l_u,  o = sum_u 2^(m_u - M) o_u / l.
// ---------------------------------------------------------------------------
// 128 threads and at most 72 registers (D <= 128): 28 warps per SM, so the
// 4096 (pair, column) warps of 32 requests x 8 KV heads x 16 columns are all
// resident at once instead of in two waves.
constexpr int kMergeThreads = 128;
template <int D, int G, bool MULTI>
__global__ void __launch_bounds__(kMergeThreads, D <= 128 ? 7 : 4)
    merge_split_kernel(const DecodeArgs a, int check_Hq, int check_dtype) {
  constexpr int PER = D / 32;
  if (threadIdx.x == 0) grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int NHG = a.head_groups;
  const long long pp = wid / G;  // pair index s * NHG + hg
  const int c = static_cast<int>(wid % G);
  const int s = static_cast<int>(pp / NHG), hg = static_cast<int>(pp % NHG);
  const int T = MULTI ? a.num_q_tokens : 1;
  const int Gq = MULTI ? a.num_q_heads / a.num_kv_heads : G;
  const int ncols = MULTI ? T * Gq : G;
  // the pair's span from the plan, which the plan kernel wrote before the
  // partition kernel began, while that kernel still runs
  MergeSpan span;
  const bool split = wid < static_cast<long long>(a.num_seqs) * NHG * G && c < ncols &&
                     merge_span(a, check_Hq, check_dtype, D, s, hg, span);
  // the partition kernel before this one wrote the partial states
  grid_dependency_wait();
  if (!split) return;
  float M, L, acc[PER];
  merge_pieces<D, G, MULTI>(a, span, c, lane, M, L, acc);
  const OutMap om{(static_cast<size_t>(s) * T * a.num_q_heads + static_cast<size_t>(hg) * Gq) * D,
                  static_cast<size_t>(a.num_q_heads) * D, Gq, D, ncols};
  const float inv = MULTI ? (L > 0.f ? 1.f / L : 0.f) : 1.f / L;  // 0: nothing attended
  if constexpr (MULTI) {
    if (lane == 0) om.put_lse(a.lse, c, M, L);
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) store1(a.out, a.out_dtype, om.row(c) + lane * PER + i, acc[i] * inv);
}

// Whether a later launch merges a partition launch's split pairs (instead of
// the last worker of each pair, at the launch's tail): with 16 columns, and
// with 8 in the general instantiation (several query tokens, padded columns or
// a log-sum-exp output).  Single-token 8-column decode keeps the in-kernel
// merge, which measured faster for it.
template <int G, bool MULTI>
constexpr bool merged_by_later_launch() {
  return G == 16 || (G == 8 && MULTI);
}

// After a bounded wait on tile k expired: stop computing and issue no new
// copies, but give the copies already issued into the warp's ring (tiles
// k .. k + depth - 1) a last short wait each before the CTA exits, so none
// lands in shared memory that a newly scheduled CTA already uses.  A copy
// that has not landed after that second limit is taken as lost; the status
// word reports the launch.  Out of line: it is cold, and inlined it would
// enlarge the streaming loop.
static __device__ __noinline__ void drain_ring(uint64_t* bars, int depth, int k, int ntiles) {
  for (int kk = k; kk < ntiles && kk < k + depth; ++kk)
    mbar_wait_bounded(smem_u32(&bars[kk % depth]), (kk / depth) & 1, kDrainLimitNs);
}

// ---------------------------------------------------------------------------
// Partition: persistent grid, one stream-K worker per CTA, one KV head per warp.
// ---------------------------------------------------------------------------
// One lookahead entry: s, hg | nt << 12, j, flags, new_slot, len, phys[kMaxBoxes].
constexpr int kEntryInts = 6 + kMaxBoxes;

template <class Core, int W, int DEPTH>
struct Smem {
  static constexpr int kStages = DEPTH * Core::kStageBytes;
  static constexpr int kScratch = Core::kScratchBytes;
  static constexpr int kMeta = DEPTH * int(sizeof(StageMeta));
  static constexpr int kBatchInts = kBatch * kEntryInts;
  static constexpr int kBatchB = kBatchInts * 4;
  static constexpr int kBars = DEPTH * 8;
  static constexpr int kPerWarp =
      round_up(kStages + kScratch + kMeta + kBatchB + kBars, Core::kAlign);
  static constexpr int kTotal = W * kPerWarp + Core::kAlign;  // + slack to align the base
};

constexpr int kSmemPerSM = 232448;  // dynamic shared memory of one SM available to CTAs

// Deepest ring (2..6 stages per warp) whose CTAs fit CPS to an SM.
template <class Core, int W, int CPS>
constexpr int pick_depth() {
  constexpr int lim = kSmemPerSM / CPS - (CPS > 1 ? 1024 : 0);
  return Smem<Core, W, 6>::kTotal <= lim   ? 6
         : Smem<Core, W, 5>::kTotal <= lim ? 5
         : Smem<Core, W, 4>::kTotal <= lim ? 4
         : Smem<Core, W, 3>::kTotal <= lim ? 3
                                           : 2;
}

struct TmaMaps {
  CUtensorMap k;
  CUtensorMap v;
};

// MULTI: several query tokens per request, idle padding columns, or a
// log-sum-exp output; without it the columns are exactly the G grouped heads
// of one token and the kernel has no per-column work.
template <class Core, int G, int W, int CPS, int DEPTH, bool MULTI>
__global__ void __launch_bounds__(W * 32, CPS)
    partition_kernel(const __grid_constant__ TmaMaps maps, const DecodeArgs a, int check_S,
                     int check_Hq, int check_Hkv, int check_D, int check_dtype) {
  using SM = Smem<Core, W, DEPTH>;
  constexpr int D = Core::ROWB / Core::ESZ;
  constexpr int PS = part_stride(G, D);
  extern __shared__ char smem_raw[];
  // Aligned by pointer arithmetic on the shared array itself (not through an
  // integer round trip), so every pointer derived from `base` stays in the
  // shared address space and its loads and stores compile to shared-memory
  // instructions rather than generic ones (about 4 us less per 32 x 4096
  // layer, measured).
  const uint32_t mis = smem_u32(smem_raw) & (Core::kAlign - 1);
  char* base = smem_raw + (mis ? Core::kAlign - mis : 0u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  char* wbase = base + warp * SM::kPerWarp;
  char* stages = wbase;
  float* scratch = reinterpret_cast<float*>(wbase + SM::kStages);
  StageMeta* meta = reinterpret_cast<StageMeta*>(wbase + SM::kStages + SM::kScratch);
  int32_t* bt = reinterpret_cast<int32_t*>(wbase + SM::kStages + SM::kScratch + SM::kMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(wbase + SM::kStages + SM::kScratch + SM::kMeta + SM::kBatchB);

  // A launch behind the plan kernel that writes its plan waits for it first,
  // and only then lets its own dependents be scheduled, so that they too
  // start after everything the plan kernel wrote is there.
  if (a.wait_first) grid_dependency_wait();
  // The next kernel of the stream may be scheduled now; it starts on an SM
  // as this launch's CTAs leave it.
  if (threadIdx.x == 0) grid_launch_dependents();
  // Until grid_dependency_wait() below, this launch only reads what the
  // kernel just before it does not write (plan, tables, lengths, slots, K/V
  // pool), through L2, and writes no global memory but error flags.
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  uint32_t* status = &hdr->status;
  if (__ldcg(&hdr->planned) != 1 || __ldcg(&hdr->num_seqs) != check_S || __ldcg(&hdr->num_q_heads) != check_Hq ||
      __ldcg(&hdr->num_kv_heads) != check_Hkv || __ldcg(&hdr->head_dim) != check_D ||
      __ldcg(&hdr->kv_dtype) != check_dtype || __ldcg(&hdr->num_workers) != a.num_workers ||
      __ldcg(&hdr->head_groups) != a.head_groups) {
    grid_dependency_wait();
    if (threadIdx.x == 0) record_status(status, kStatusPlanMismatch);
    return;
  }
  const long long TT = __ldcg(&hdr->total_tiles);
  const int NW = a.num_workers;
  const int v = blockIdx.x;  // this CTA's worker id; warp = head within the group
  const int4 wp = __ldcg(reinterpret_cast<const int4*>(a.ws + a.off_wplan) + 2 * v);
  const int first_len = __ldcg(reinterpret_cast<const int4*>(a.ws + a.off_wplan) + 2 * v + 1).x;
  const int ntiles = wp.y - wp.x;

  const int S = a.num_seqs, Hkv = a.num_kv_heads, NHG = a.head_groups, Bsz = a.block_size;
  const int Hq = a.num_q_heads;
  // T query tokens per request: the columns of a KV head are its Gq grouped
  // heads for each token, c = i * Gq + k, padded with idle columns up to G.
  const int T = MULTI ? a.num_q_tokens : 1;
  const int Gq = MULTI ? Hq / Hkv : G;
  const int ncols = MULTI ? T * Gq : G;
  const int gq_mul = ((1 << 16) + Gq - 1) / Gq;  // exact division of column indices < 16 by Gq
  const int box_rows = Bsz < kTile ? Bsz : kTile;
  const int nbox = kTile / box_rows;  // boxes per tile per chunk
  const uint64_t pol = policy_evict_first();
  float* partials = reinterpret_cast<float*>(a.ws + a.off_partials);
  int32_t* counters = reinterpret_cast<int32_t*>(a.ws + a.off_counters);

  if (ntiles > 0 && ncols < G) {
    // idle columns read zeros: the bulk copies fill only the first ncols q rows
    for (int st = 0; st < DEPTH; ++st)
      for (int i = ncols * Core::ROWB / 16 + lane; i < Core::QB / 16; i += 32)
        reinterpret_cast<uint4*>(stages + st * Core::kStageBytes + Core::kQOff)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if constexpr (MULTI) {
    if (threadIdx.x == 0) s_lse_out = a.lse;
  }
  if (ntiles > 0 && lane == 0) {
    for (int i = 0; i < DEPTH; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  // Block-table lookahead, one batch ahead: walk() finds (s, hg, j) of the
  // next kBatch tiles (lane l takes tile kb + l) and starts their table loads
  // into registers; commit() stores them to shared memory one batch later,
  // when the loads have long landed.  The cursor (request cs, offset coff in
  // its NHG * nt tiles, its length clen) is warp-uniform; seq_lens is only
  // read when the walk crosses into a new request.
  int cs = wp.z, coff = wp.w;
  int clen = first_len;
  int n_s = 0, n_hg = 0, n_j = 0, n_flags = 0, n_nt = 0, n_len = 0;
  long long n_slot = -1;
  int n_phys[kMaxBoxes];
  uint32_t n_have = 0, n_over = 0;  // bit b: box b is read / box b lies past the table row
  bool n_valid = false;

  auto walk = [&](int kb) {
    n_valid = lane < kBatch && kb + lane < ntiles;
    n_have = 0;
    n_over = 0;
    if (n_valid) {
      int s = cs, off = coff + lane, len = clen;
      int nt = ntiles_of(len);
      while (off >= NHG * nt) {
        off -= NHG * nt;
        if (s + 1 >= S) {  // inconsistent with the plan: stop here
          record_status(status, kStatusPlanMismatch);
          off = 0;
          break;
        }
        ++s;
        len = __ldcg(a.seq_lens + s);
        nt = ntiles_of(len);
      }
      const int hg = nt > 0 ? off / nt : 0;
      const int j = nt > 0 ? off % nt : 0;
      const int nblk = (len + Bsz - 1) / Bsz;
      const int lb0 = (j * kTile) / Bsz;
      n_s = s;
      n_hg = hg;
      n_j = j;
      n_nt = nt;
      n_flags = (min(kTile, len - j * kTile) << 8) | (j == nt - 1 ? 2 : 0);
      n_len = len;
      n_slot = (a.new_slots != nullptr && j == nt - 1) ? __ldcg(a.new_slots + s) : -1;
      const int32_t* row = a.block_tables + static_cast<size_t>(s) * a.max_blocks;
#pragma unroll
      for (int b = 0; b < kMaxBoxes; ++b) {
        n_phys[b] = -1;
        if (b < nbox && lb0 + b < nblk) {
          if (lb0 + b >= a.max_blocks) {
            n_over |= 1u << b;
          } else {
            n_phys[b] = __ldcg(row + lb0 + b);
            n_have |= 1u << b;
          }
        }
      }
      cs = s;
      coff = off + 1;
      clen = len;
    }
    // the cursor for the next batch comes from the batch's last lane
    cs = __shfl_sync(0xffffffffu, cs, kBatch - 1);
    coff = __shfl_sync(0xffffffffu, coff, kBatch - 1);
    clen = __shfl_sync(0xffffffffu, clen, kBatch - 1);
  };

  auto commit = [&]() {
    if (n_valid) {
      int32_t* e = bt + lane * kEntryInts;
      e[0] = n_s;
      e[1] = n_hg | (n_nt << 12);
      e[2] = n_j;
      e[3] = n_flags;
      e[4] = -1;
      if (n_slot >= static_cast<long long>(a.num_blocks) * Bsz)
        record_status(status, kStatusBadTable);  // new-token slot outside the pool: not written
      else if (n_slot >= 0)
        e[4] = static_cast<int>(n_slot);
      if constexpr (MULTI) e[5] = n_len;
#pragma unroll
      for (int b = 0; b < kMaxBoxes; ++b) {
        int phys = -1;
        if (n_over & (1u << b)) {
          record_status(status, kStatusBadTable);  // length beyond the table row
        } else if (n_have & (1u << b)) {
          phys = n_phys[b];
          if (phys < 0 || phys >= a.num_blocks) {
            record_status(status, kStatusBadTable);
            phys = a.num_blocks;  // out of the tensor map: TMA fills zeros
          }
        }
        e[6 + b] = phys;
      }
    }
    __syncwarp();
  };

  int last_s = -1, last_hg = -1;
  // q is written by earlier kernels: in the prologue (before the dependency
  // wait) a stage's q copy is held back, and the stage's arrival with it.
  bool defer_q = true;
  uint32_t q_pending = 0;  // lane 0: stages whose q copy and arrival wait
  auto load_q = [&](int st, int s, int head) {
    char* stage = stages + st * Core::kStageBytes;
    const uint32_t bar = smem_u32(&bars[st]);
    // the pair's G columns: Gq grouped heads of each of the T query tokens
    for (int i = 0; i < T; ++i) {
      const char* qsrc = reinterpret_cast<const char*>(a.q) +
                         ((static_cast<size_t>(s) * T + i) * Hq + static_cast<size_t>(head) * Gq) * Core::ROWB;
      bulk_load(smem_u32(stage + Core::kQOff + i * Gq * Core::ROWB), qsrc, Gq * Core::ROWB, bar);
    }
  };
  auto issue = [&](int k) {
    if ((k % kBatch) == 0) {
      commit();               // batch k, loaded during the previous batch
      walk(k + kBatch);       // start loading batch k + kBatch
    }
    if (lane == 0) {
      const int32_t* e = bt + (k % kBatch) * kEntryInts;
      const int s = e[0], hg = e[1] & 0xfff, j = e[2];
      const int head = hg * W + warp;
      const bool newpair = (s != last_s) || (hg != last_hg);
      last_s = s;
      last_hg = hg;
      const int st = k % DEPTH;
      char* stage = stages + st * Core::kStageBytes;
      meta[st].s = s;
      meta[st].hg = hg;
      meta[st].j = j;
      meta[st].flags = e[3] | (newpair ? 1 : 0);
      meta[st].nt = e[1] >> 12;
      meta[st].new_slot = e[4];
      if constexpr (MULTI) meta[st].len = e[5];
      const uint32_t bar = smem_u32(&bars[st]);
      int nb = 0;
#pragma unroll
      for (int b = 0; b < kMaxBoxes; ++b) nb += (b < nbox && e[6 + b] >= 0) ? 1 : 0;
      const uint32_t box_bytes = static_cast<uint32_t>(box_rows * Core::kChunkRowBytes);
      uint32_t bytes = 2u * nb * Core::kChunks * box_bytes;
      if (newpair) bytes += ncols * Core::ROWB;
      fence_proxy_async_smem();
      if (newpair && defer_q) {
        mbar_expect_tx(bar, bytes);  // arrival after the q copy, past the dependency wait
        q_pending |= 1u << st;
      } else {
        mbar_arrive_expect_tx(bar, bytes);
        if (newpair) load_q(st, s, head);
      }
      const int slot0 = Bsz >= kTile ? (j * kTile) % Bsz : 0;
      if (tile_map_5d(Core::ROWB, Core::kChunkRowBytes, box_rows, Core::kSwizzle, Core::kBlockRows)) {
        if (box_rows == kTile) {
          // one 5-D box per tile: all 128-byte parts of its 16 rows (two copy
          // instructions per tile instead of four; 0.5 us less per layer, measured)
          const int phys = e[6];
          if (phys >= 0) {
            tma_load_5d(smem_u32(stage + Core::kKOff), &maps.k, 0, slot0, 0, head, phys, bar, pol);
            tma_load_5d(smem_u32(stage + Core::kVOff), &maps.v, 0, slot0, 0, head, phys, bar, pol);
          }
        } else {
          // one box per block, all parts of its rows, block after block
          // (the core's [block][part][row] layout; each box 1 KiB-aligned)
#pragma unroll 1
          for (int b = 0; b < nbox; ++b) {
            const int phys = e[6 + b];
            if (phys >= 0) {
              const uint32_t off = b * box_rows * Core::ROWB;
              tma_load_5d(smem_u32(stage + Core::kKOff + off), &maps.k, 0, 0, 0, head, phys, bar, pol);
              tma_load_5d(smem_u32(stage + Core::kVOff + off), &maps.v, 0, 0, 0, head, phys, bar, pol);
            }
          }
        }
      } else {
        // A runtime loop over the tile's boxes: an unrolled loop over the
        // four a tile can have put four boxes' worth of predicated copy
        // instructions and their operand moves into every tile (about 5 us
        // more per 32 x 4096 layer, measured).
#pragma unroll 1
        for (int b = 0; b < nbox; ++b) {
          const int phys = e[6 + b];
          if (phys >= 0) {
#pragma unroll
            for (int c = 0; c < Core::kChunks; ++c) {
              const uint32_t off = c * Core::kChunkBytes + b * box_bytes;
              tma_load_4d(smem_u32(stage + Core::kKOff + off), &maps.k, c * Core::kBoxInner, slot0, head,
                          phys, bar, pol);
              tma_load_4d(smem_u32(stage + Core::kVOff + off), &maps.v, c * Core::kBoxInner, slot0, head,
                          phys, bar, pol);
            }
          }
        }
      }
    }
    __syncwarp();
  };

  if (ntiles > 0) {
    walk(0);
    const int prologue = ntiles < DEPTH ? ntiles : DEPTH;
    for (int k = 0; k < prologue; ++k) issue(k);
  }
  // Everything below may read what earlier kernels wrote (q, k_new, v_new)
  // and writes global memory.
  grid_dependency_wait();
  defer_q = false;
  if (lane == 0) {
    for (int st = 0; st < DEPTH; ++st) {
      if (q_pending & (1u << st)) {
        load_q(st, meta[st].s, meta[st].hg * W + warp);
        mbar_arrive(smem_u32(&bars[st]));
      }
    }
  }
  __syncwarp();

  // Requests of length 0 produce zeros; CTA v writes those of pairs v, v + NW, ...
  for (long long p = v; p < static_cast<long long>(S) * NHG; p += NW) {
    const int s = static_cast<int>(p / NHG), hg = static_cast<int>(p % NHG);
    if (a.seq_lens[s] != 0) continue;
    const OutMap om{(static_cast<size_t>(s) * T * Hq + static_cast<size_t>(hg * W + warp) * Gq) * D,
                    static_cast<size_t>(Hq) * D, Gq, D, ncols};
    for (int i = lane; i < ncols * D; i += 32) store1(a.out, a.out_dtype, om.row(i / D) + i % D, 0.f);
    if constexpr (MULTI) {
      if (lane < ncols) om.put_lse(a.lse, lane, -INFINITY, 0.f);
    }
  }
  if (ntiles <= 0) return;

  typename Core::State state;
  bool have = false;
  int ps = 0, phg = 0, jfirst = 0, pnt = 0;
  long long pstart = 0;
  bool last_is_end = false;

  auto flush = [&](bool final) {
    const int head = phg * W + warp;
    const OutMap om{(static_cast<size_t>(ps) * T * Hq + static_cast<size_t>(head) * Gq) * D,
                    static_cast<size_t>(Hq) * D, Gq, D, ncols};
    float* const lse = MULTI ? a.lse : nullptr;
    if (jfirst == 0 && last_is_end) {  // the whole pair is in this CTA's range
      Core::finish(state, true, a.out, a.out_dtype, om, nullptr, lane, lse);
      return;
    }
    const long long pp = static_cast<long long>(ps) * NHG + phg;  // pair index
    float* part = partials + (static_cast<size_t>(v + pp) * W + warp) * PS;
    Core::finish(state, false, a.out, a.out_dtype, om, part, lane);
    // a later launch merges the pieces (merge_split_kernel right behind this
    // kernel, or the shared-prefix call's combine), no counting in
    if constexpr (merged_by_later_launch<G, MULTI>()) return;
    // Count this CTA in for (request, KV head).  The pair's counter holds two
    // fields: the low 16 bits count pieces that ended their CTA's range, the
    // high 16 bits the one piece a range can hold before that (the tail of a
    // pair begun by an earlier CTA, flushed mid-range when the warp moves on).
    // The mid-range piece counts in with a reduction that returns nothing
    // (release: its partial writes are visible first), so the stream does not
    // stall on a round trip.  Pieces at the end of a range count in with an
    // acquire-release atomic; the last of those merges, first waiting, if it
    // has not arrived yet, for the mid-range piece (rare: that piece is the
    // first its CTA computes).
    const size_t ctr = static_cast<size_t>(ps) * Hkv + head;
    __syncwarp();
    if (!final) {
      if (lane == 0) red_release_gpu_add(reinterpret_cast<unsigned*>(&counters[ctr]), 1u << 16);
      return;
    }
    const int v0 = owner_of(pstart, TT, NW), v1 = owner_of(pstart + pnt - 1, TT, NW);
    int expected = v1 - v0 + 1;  // with TT >= NW every CTA owns at least one tile
    if (TT < NW) {
      expected = 0;
      for (int u = v0; u <= v1; ++u) expected += range_begin(u, TT, NW) < range_begin(u + 1, TT, NW) ? 1 : 0;
    }
    // the pair's last piece is flushed mid-range when its CTA's range goes on
    // past the pair's end
    const int expected_mid = (v1 != v0 && range_begin(v1 + 1, TT, NW) > pstart + pnt) ? 1 : 0;
    // The only piece flushed at a range end (the pair's other piece is the
    // mid-range one, the common case for short pairs) merges whenever the
    // mid-range piece counts in, so it counts nothing in itself: no atomic,
    // and no wait for its own partial writes, which only this warp reads.
    const bool sole = expected - expected_mid == 1;
    int prev = 0;
    if (!sole) {
      if (lane == 0) prev = atomic_add_acq_rel_gpu(&counters[ctr], 1);
      prev = __shfl_sync(0xffffffffu, prev, 0);
    }
    if (sole || (prev & 0xffff) == expected - expected_mid - 1) {
      if ((prev >> 16) < expected_mid) {
        // bounded wait for the mid-range piece (its CTA is running or about
        // to: it needs nothing from this one)
        bool ok = false;
        if (lane == 0) {
          const uint64_t t0 = globaltimer();
          while (!ok) {
            ok = (ld_acquire_gpu(reinterpret_cast<const unsigned*>(&counters[ctr])) >> 16) >= unsigned(expected_mid);
            if (!ok && globaltimer() - t0 > kWaitLimitNs) break;
            if (!ok) __nanosleep(64);
          }
          if (!ok) record_status(status, kStatusTimeout);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) return;
      }
      __syncwarp();
      merge_pair<D, G, W, MULTI>(partials, pp, warp, v0, v1, TT, NW, a.out, a.out_dtype, om, lane);
      if (lane == 0) atomicExch(&counters[ctr], 0);
    }
  };

  for (int k = 0; k < ntiles; ++k) {
    const int st = k % DEPTH;
    if (!mbar_wait_bounded(smem_u32(&bars[st]), (k / DEPTH) & 1)) {
      if (lane == 0) record_status(status, kStatusTimeout);
      drain_ring(bars, DEPTH, k, ntiles);
      return;
    }
    const StageMeta m = meta[st];
    const char* stage = stages + st * Core::kStageBytes;
    if (m.flags & 1) {
      if (have) flush(false);
      have = true;
      ps = m.s;
      phg = m.hg;
      jfirst = m.j;
      pnt = m.nt;
      pstart = static_cast<long long>(wp.x) + k - m.j;
      Core::begin_pair(state, stage + Core::kQOff, a.scale_log2, lane);
    }
    const int nvalid = m.flags >> 8;
    last_is_end = (m.flags & 2) != 0;
    if (m.new_slot >= 0) {
      // Folded append: this tile holds the pair's new token (row nvalid - 1).
      // Write its K and V row to the pool and over the stale tile row.
      const int head = m.hg * W + warp;
      constexpr int U = Core::ROWB / 16;
      const size_t src_off = (static_cast<size_t>(m.s) * Hkv + head) * Core::ROWB;
      const size_t dst_off = (static_cast<size_t>(m.new_slot) * Hkv + head) * Core::ROWB;
      for (int i = lane; i < 2 * U; i += 32) {
        const bool is_v = i >= U;
        const int unit = is_v ? i - U : i;
        const uint4 val = *reinterpret_cast<const uint4*>(
            static_cast<const char*>(is_v ? a.v_new : a.k_new) + src_off + unit * 16);
        *reinterpret_cast<uint4*>(static_cast<char*>(is_v ? a.v_pool : a.k_pool) + dst_off + unit * 16) = val;
        *reinterpret_cast<uint4*>(const_cast<char*>(stage) + (is_v ? Core::kVOff : Core::kKOff) +
                                  Core::row_unit(nvalid - 1, unit)) = val;
      }
      __syncwarp();
    }
    const TileLim<MULTI> lim{nvalid, MULTI ? m.len - m.j * kTile : nvalid, T, gq_mul, a.causal};
    if constexpr (Core::kSwizzle) {
      Core::tile(state, stage + Core::kKOff, stage + Core::kVOff, lim, a.scale_log2, lane);
    } else {
      Core::tile(state, stage + Core::kKOff, stage + Core::kVOff, lim, scratch, lane);
    }
    __syncwarp();
    if (k + DEPTH < ntiles) issue(k + DEPTH);
  }
  if (have) flush(true);
}


// ---------------------------------------------------------------------------
// Host-side launch helpers
// ---------------------------------------------------------------------------
struct Geometry {
  int S, Hq, Hkv, G, D, dtype;
  int HG, NHG, CPS, NW;
  WsLayout lay;
  bool overlap = false;  // launch as a programmatic dependent launch
};

extern int g_kernel_choice;  // 0 auto, 1 CUDA-core tiles, 2 tensor-core tiles (bf16)

bool make_pool_map(CUtensorMap* m, const void* pool, int dtype, int D, int B, int Hkv, int N,
                   int box_inner, int box_rows, bool swizzle, int block_rows);

template <class Core, int G, int W, int CPS, bool MULTI>
int launch_partition(const Geometry& geo, const DecodeArgs& args, const void* k_pool, const void* v_pool,
                     cudaStream_t stream) {
  constexpr int DEPTH = pick_depth<Core, W, CPS>();
  using SM = Smem<Core, W, DEPTH>;
  static_assert(SM::kTotal <= kSmemPerSM, "shared memory budget");
  TmaMaps maps;
  const int box_rows = args.block_size < kTile ? args.block_size : kTile;
  // a core that lays tiles out block by block reads only boxes of its rows
  if (Core::kBlockRows != kTile && box_rows != Core::kBlockRows) return PKV_ERR_INVALID;
  if (!make_pool_map(&maps.k, k_pool, geo.dtype, geo.D, args.block_size, geo.Hkv, args.num_blocks,
                     Core::kBoxInner, box_rows, Core::kSwizzle, Core::kBlockRows) ||
      !make_pool_map(&maps.v, v_pool, geo.dtype, geo.D, args.block_size, geo.Hkv, args.num_blocks,
                     Core::kBoxInner, box_rows, Core::kSwizzle, Core::kBlockRows)) {
    host::set_error("cuTensorMapEncodeTiled failed");
    return PKV_ERR_CUDA;
  }
  auto kern = partition_kernel<Core, G, W, CPS, DEPTH, MULTI>;
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal);
    if (e != cudaSuccess) return host::cuda_fail(e);
    configured_dev = dev;
  }
  if (!geo.overlap) {
    kern<<<geo.NW, W * 32, SM::kTotal, stream>>>(maps, args, geo.S, geo.Hq, geo.Hkv, geo.D, geo.dtype);
    return host::check_launch();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(geo.NW);
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = SM::kTotal;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, maps, args, geo.S, geo.Hq, geo.Hkv, geo.D, geo.dtype);
  if (e != cudaSuccess) return host::cuda_fail(e);
  return host::check_launch();
}

// The merge kernel of a 16-column launch, as a programmatic dependent launch
// behind the partition kernel: one warp per (pair, column).
template <int D, int G, bool MULTI>
int launch_merge(const Geometry& geo, const DecodeArgs& args, cudaStream_t stream) {
  const long long warps = static_cast<long long>(args.num_seqs) * args.head_groups * G;
  if (warps == 0) return PKV_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((warps * 32 + kMergeThreads - 1) / kMergeThreads));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the plan's head count (padded to the column group for several query tokens)
  const cudaError_t e = cudaLaunchKernelEx(&cfg, merge_split_kernel<D, G, MULTI>, args, geo.Hq, geo.dtype);
  if (e != cudaSuccess) return host::cuda_fail(e);
  return host::check_launch();
}

template <class Core, int G>
int launch_core(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
                cudaStream_t stream) {
  constexpr int WPS = (Core::ROWB >= 512) ? 4 : 8;
  constexpr int D = Core::ROWB / Core::ESZ;
  if (geo.HG != 1) return PKV_ERR_INVALID;
  const bool multi = args.num_q_tokens > 1 || args.num_q_heads != G * args.num_kv_heads || args.lse != nullptr;
  const int rc = multi ? launch_partition<Core, G, 1, WPS, true>(geo, args, k, v, stream)
                       : launch_partition<Core, G, 1, WPS, false>(geo, args, k, v, stream);
  if (rc != PKV_OK || args.merge_by_caller) return rc;
  if constexpr (G == 16) {
    return multi ? launch_merge<D, G, true>(geo, args, stream) : launch_merge<D, G, false>(geo, args, stream);
  } else if constexpr (G == 8) {
    if (multi) return launch_merge<D, G, true>(geo, args, stream);  // merged_by_later_launch<8, true>
  }
  return rc;
}

// One (storage type, head_dim): dispatch on the group size and the core.
template <typename T, int D>
int run_decode(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
               cudaStream_t stream) {
  auto per_g = [&](auto gc) -> int {
    constexpr int G = decltype(gc)::value;
    // tensor-core tiles for bf16: up to 8 columns with the tokens in the MMA's
    // M dimension; 16 columns (head_dim <= 128) with the columns in M.  Block
    // size 4 (head_dim >= 128): tiles laid out block by block.
    if constexpr (sizeof(T) == 2 && G <= 8) {
      if (args.block_size >= 8 && g_kernel_choice != 1)
        return launch_core<MmaCore<D, G>, G>(geo, args, k, v, stream);
      if constexpr (D >= 128) {
        if (args.block_size == 4 && g_kernel_choice != 1)
          return launch_core<MmaCore<D, G, 4>, G>(geo, args, k, v, stream);
      }
    }
    if constexpr (sizeof(T) == 2 && G == 16 && D <= 128) {
      if (args.block_size >= 8 && g_kernel_choice != 1)
        return launch_core<MmaCoreM16<D>, G>(geo, args, k, v, stream);
      if constexpr (D >= 128) {
        if (args.block_size == 4 && g_kernel_choice != 1)
          return launch_core<MmaCoreM16<D, 4>, G>(geo, args, k, v, stream);
      }
    }
    return launch_core<FmaCore<T, D, G>, G>(geo, args, k, v, stream);
  };
  switch (geo.G) {
    case 1: return per_g(std::integral_constant<int, 1>{});
    case 2: return per_g(std::integral_constant<int, 2>{});
    case 4: return per_g(std::integral_constant<int, 4>{});
    case 8: return per_g(std::integral_constant<int, 8>{});
    case 16: return per_g(std::integral_constant<int, 16>{});
  }
  return PKV_ERR_INVALID;
}

int run_bf16_64(const Geometry&, const DecodeArgs&, const void*, const void*, cudaStream_t);
int run_bf16_128(const Geometry&, const DecodeArgs&, const void*, const void*, cudaStream_t);
int run_bf16_256(const Geometry&, const DecodeArgs&, const void*, const void*, cudaStream_t);
int run_f32_64(const Geometry&, const DecodeArgs&, const void*, const void*, cudaStream_t);
int run_f32_128(const Geometry&, const DecodeArgs&, const void*, const void*, cudaStream_t);

}  // namespace pkv
