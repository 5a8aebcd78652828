// Decode attention entry points of libpkv: the plan kernel, the host side that
// validates arguments and builds the TMA tensor maps, and the C ABI.  The
// partition kernel (persistent stream-K over one-warp CTAs, each taking an
// equal range of (request, KV head, 16-token tile) units; the last CTA on a
// split (request, KV head) merges the partial states) lives in
// pkv_decode_kernels.cuh and is instantiated per (storage type, head_dim) in
// pkv_decode_<type>_<d>.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/pkv.h"
#include "pkv_decode_kernels.cuh"
#include "pkv_host.h"

namespace pkv {

// ---------------------------------------------------------------------------
// Plan: tiles per request (prefix), each worker's starting position, and the
// arrival counters cleared.  One CTA: a block scan over the requests, then one
// binary search per worker.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kPlanSmemSeqs = 8192;  // prefix kept in shared memory up to this many requests

// len_of(s): the length of request s (read from an array, or computed).
template <class LenOf>
__device__ __forceinline__ void plan_body(LenOf len_of, int S, int Hq, int Hkv,
                                          int NHG, int D, int kv_dtype, int NW, char* ws, size_t off_prefix,
                                          size_t off_wplan, size_t off_counters) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  int32_t* prefix = reinterpret_cast<int32_t*>(ws + off_prefix);
  int4* wplan = reinterpret_cast<int4*>(ws + off_wplan);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + off_counters);
  __shared__ long long warp_tot[kPlanThreads / 32];
  __shared__ long long total_sh;
  __shared__ int32_t sp[kPlanSmemSeqs + 1];
  const bool in_smem = S <= kPlanSmemSeqs;

  const int tid = threadIdx.x;
  const int chunk = (S + kPlanThreads - 1) / kPlanThreads;
  const int s0 = min(S, tid * chunk), s1 = min(S, s0 + chunk);
  long long local = 0;
  for (int s = s0; s < s1; ++s) local += ntiles_of(len_of(s));
  // block exclusive scan of `local`
  const int lane = tid & 31, warp = tid >> 5;
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const long long w = warp_tot[lane];
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of the warp totals
    if (lane == 31) total_sh = wi;
  }
  __syncthreads();
  long long run = warp_tot[warp] + incl - local;
  for (int s = s0; s < s1; ++s) {
    prefix[s] = static_cast<int32_t>(run);
    if (in_smem) sp[s] = static_cast<int32_t>(run);
    run += ntiles_of(len_of(s));
  }
  const long long total_seq_tiles = total_sh;
  if (tid == 0) {
    prefix[S] = static_cast<int32_t>(total_seq_tiles);
    if (in_smem) sp[S] = static_cast<int32_t>(total_seq_tiles);
  }
  for (long long p = tid; p < static_cast<long long>(S) * Hkv; p += kPlanThreads) counters[p] = 0;
  __syncthreads();
  const long long T = total_seq_tiles * NHG;
  const int32_t* P = in_smem ? sp : prefix;

  // Worker v owns tiles [floor(v T / NW), floor((v+1) T / NW)); its first
  // request is the last s with NHG * P[s] <= start (skipping empty requests).
  for (int v = tid; v < NW; v += kPlanThreads) {
    if (T == 0) {
      wplan[2 * v] = make_int4(0, 0, 0, 0);
      wplan[2 * v + 1] = make_int4(0, 0, 0, 0);
      continue;
    }
    const long long a = range_begin(v, T, NW);
    const long long b = range_begin(v + 1, T, NW);
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<long long>(P[mid]) * NHG <= a) lo = mid; else hi = mid - 1;
    }
    wplan[2 * v] = make_int4(static_cast<int>(a), static_cast<int>(b), lo,
                             static_cast<int>(a - static_cast<long long>(P[lo]) * NHG));
    wplan[2 * v + 1] = make_int4(len_of(lo), 0, 0, 0);  // saves the worker a dependent load
  }
  if (tid == 0) {
    hdr->num_seqs = S;
    hdr->num_q_heads = Hq;
    hdr->num_kv_heads = Hkv;
    hdr->head_dim = D;
    hdr->kv_dtype = kv_dtype;
    hdr->num_workers = NW;
    hdr->head_groups = NHG;
    hdr->total_tiles = T;
    hdr->planned = 1;
  }
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ seq_lens,
                                                            int S, int Hq, int Hkv, int NHG, int D,
                                                            int kv_dtype, int NW, char* ws,
                                                            size_t off_prefix, size_t off_wplan,
                                                            size_t off_counters) {
  // an attention launch after this one may be scheduled now: it waits for
  // this kernel before reading the plan
  if (threadIdx.x == 0) grid_launch_dependents();
  plan_body([seq_lens](int s) { return seq_lens[s]; }, S, Hq, Hkv, NHG, D, kv_dtype, NW, ws, off_prefix,
            off_wplan, off_counters);
}

}  // namespace pkv

// ===========================================================================
// Host side
// ===========================================================================
namespace pkv {

int g_kernel_choice = 0;
int g_launch_overlap = 0;

namespace {
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                              CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                              CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}
}  // namespace

// Pool viewed as 4-D (d, slot, kv head, block), box (inner, rows, 1, 1); or,
// for 16-row boxes of swizzled rows longer than one 128-byte part, as 5-D
// (inner part of d, slot, part, kv head, block) with one box per tile.
bool make_pool_map(CUtensorMap* m, const void* pool, int dtype, int D, int B, int Hkv, int N,
                   int box_inner, int box_rows, bool swizzle, int block_rows) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = dtype == PKV_BF16 ? 2 : 4;
  if (tile_map_5d(D * static_cast<int>(es), box_inner * static_cast<int>(es), box_rows, swizzle, block_rows)) {
    // (inner part of d, slot, part of d, kv head, block): one box fetches all
    // parts of d of a 16-row tile, part-major, as the 4-D map's boxes would,
    // or of one block's box_rows rows
    const cuuint64_t parts = static_cast<cuuint64_t>(D / box_inner);
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(box_inner), static_cast<cuuint64_t>(B), parts,
                          static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[4] = {es * Hkv * D, es * box_inner, es * D, es * Hkv * D * B};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows),
                         static_cast<cuuint32_t>(parts), 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    5, const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
  }
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(B),
                        static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[3] = {es * Hkv * D, es * D, es * Hkv * D * B};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  4, const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace pkv

namespace {

using namespace pkv;

int num_sms_current() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 0 || dev >= 64) return -1;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev] = n;
  }
  return cache[dev];
}

bool valid_dtype(int d) { return d == PKV_BF16 || d == PKV_F32; }
int esize(int d) { return d == PKV_BF16 ? 2 : 4; }

bool shape_ok(int Hq, int Hkv, int D, int dtype) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || Hkv >= 4096) return false;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return false;
  if (dtype == PKV_BF16) return D == 64 || D == 128 || D == 256;
  if (dtype == PKV_F32) return D == 64 || D == 128;
  return false;
}

// Workers per SM: 8 for rows of up to 256 bytes, 4 for 512-byte rows (their
// stages are twice as large).  Each worker is a one-warp CTA (head group of
// one KV head): measured on the 32 x 4096 decode, one-warp workers stream
// faster than CTAs whose warps share a block's KV heads (102 vs 110 us per
// layer), so the head-group width is 1.  The plan and every kernel variant
// agree on these numbers.
int warps_per_sm(int D, int dtype) { return D * esize(dtype) >= 512 ? 4 : 8; }
int head_group(int /*Hkv*/, int /*wps*/) { return 1; }

bool geometry(int S, int Hq, int Hkv, int D, int dtype, Geometry* g) {
  if (S < 0 || !valid_dtype(dtype) || !shape_ok(Hq, Hkv, D, dtype)) return false;
  const int sms = num_sms_current();
  if (sms <= 0) return false;
  const int wps = warps_per_sm(D, dtype);
  const int HG = head_group(Hkv, wps);
  const int CPS = wps / HG;
  const int NW = sms * CPS;
  *g = Geometry{S, Hq, Hkv, Hq / Hkv, D, dtype, HG, Hkv / HG, CPS, NW,
                WsLayout(S, Hkv, HG, Hq / Hkv, D, NW)};
  return true;
}

// Query heads of the plan for T tokens per request: H_kv * P with P the
// smallest power of two >= T * G (columns per KV head); 0 if unsupported.
int32_t multi_query_heads(int32_t T, int32_t Hq, int32_t Hkv) {
  if (T < 1 || T > 16 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return 0;
  const int cols = T * (Hq / Hkv);
  if (cols > 16) return 0;
  int P = 1;
  while (P < cols) P <<= 1;
  return Hkv * P;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int do_plan(const Geometry& geo, const int32_t* seq_lens, void* ws, cudaStream_t stream) {
  plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, geo.S, geo.Hq, geo.Hkv, geo.NHG, geo.D, geo.dtype,
                                              geo.NW, static_cast<char*>(ws), geo.lay.prefix,
                                              geo.lay.wplan, geo.lay.counters);
  return host::check_launch();
}

int check_common(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                 int32_t max_blocks, const int32_t* seq_lens, int32_t S, int32_t B, int32_t N,
                 const void* out, int32_t out_dtype, const void* ws, size_t ws_bytes,
                 const Geometry& geo) {
  if (B != 4 && B != 8 && B != 16 && B != 32 && B != 64 && B != 128 && B != 256) return PKV_ERR_INVALID;
  if (N <= 0 || max_blocks < 0 || !valid_dtype(out_dtype)) return PKV_ERR_INVALID;
  if (S > 0 && (!q || !k_pool || !v_pool || !block_tables || !seq_lens || !out)) return PKV_ERR_INVALID;
  if (!ws || !aligned(ws, 256) || ws_bytes < geo.lay.total) return PKV_ERR_INVALID;
  if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(q, 16) || !aligned(out, 16))
    return PKV_ERR_INVALID;
  // flattened tile indices are int32; tiles per request are packed in 19 bits
  const long long max_tiles_seq = (static_cast<long long>(max_blocks) * B + kTile - 1) / kTile;
  if (static_cast<long long>(S) * geo.NHG * max_tiles_seq >= (1ll << 31)) return PKV_ERR_INVALID;
  if (max_tiles_seq >= (1ll << 19)) return PKV_ERR_INVALID;
  return PKV_OK;
}

}  // namespace

extern "C" {

size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim) {
  Geometry g;
  // the layout depends on the storage type only through the worker count;
  // size for the larger of the two.
  size_t best = 0;
  for (int dt : {PKV_BF16, PKV_F32}) {
    if (geometry(num_seqs, num_q_heads, num_kv_heads, head_dim, dt, &g) && g.lay.total > best)
      best = g.lay.total;
  }
  return best;
}

size_t pkv_multi_query_workspace_bytes(int32_t num_seqs, int32_t num_q_tokens, int32_t num_q_heads,
                                       int32_t num_kv_heads, int32_t head_dim) {
  const int32_t hq_eff = multi_query_heads(num_q_tokens, num_q_heads, num_kv_heads);
  if (hq_eff <= 0) return 0;
  return pkv_decode_workspace_bytes(num_seqs, hq_eff, num_kv_heads, head_dim);
}

int pkv_decode_plan(const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                    int32_t num_kv_heads, int32_t head_dim, int32_t kv_dtype, void* workspace,
                    size_t workspace_bytes, pkv_stream_t stream) {
  Geometry geo;
  if (!geometry(num_seqs, num_q_heads, num_kv_heads, head_dim, kv_dtype, &geo)) return PKV_ERR_INVALID;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < geo.lay.total) return PKV_ERR_INVALID;
  if (num_seqs > 0 && !seq_lens) return PKV_ERR_INVALID;
  return do_plan(geo, seq_lens, workspace, static_cast<cudaStream_t>(stream));
}

namespace {

int run_impl(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
             int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
             int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
             int32_t kv_dtype, void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
             pkv_stream_t stream, const void* k_new, const void* v_new, const int64_t* new_slots,
             int32_t num_q_tokens = 1, bool overlap = false, int32_t causal = 1, float* lse = nullptr,
             bool after_plan = false, bool merge_by_caller = false, DecodeArgs* args_out = nullptr) {
  // T query tokens per request run as more grouped heads over the same KV
  // heads: the columns of a KV head are (query token, grouped head), padded
  // to a power of two.
  if (new_slots && num_q_tokens != 1) return PKV_ERR_INVALID;
  const int32_t hq_eff = multi_query_heads(num_q_tokens, num_q_heads, num_kv_heads);
  if (hq_eff <= 0) return PKV_ERR_INVALID;
  Geometry geo;
  if (!geometry(num_seqs, hq_eff, num_kv_heads, head_dim, kv_dtype, &geo)) return PKV_ERR_INVALID;
  int rc = check_common(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                        block_size, num_blocks, out, out_dtype, workspace, workspace_bytes, geo);
  if (rc != PKV_OK) return rc;
  if (!std::isfinite(scale)) return PKV_ERR_INVALID;
  if (new_slots) {
    if (num_seqs > 0 && (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)))
      return PKV_ERR_INVALID;
    if (static_cast<long long>(num_blocks) * block_size >= (1ll << 31)) return PKV_ERR_INVALID;
  }
  if (num_seqs == 0) return PKV_OK;
  DecodeArgs args{};
  args.q = q;
  args.block_tables = block_tables;
  args.seq_lens = seq_lens;
  args.out = out;
  args.ws = static_cast<char*>(workspace);
  args.off_prefix = geo.lay.prefix;
  args.off_wplan = geo.lay.wplan;
  args.off_counters = geo.lay.counters;
  args.off_partials = geo.lay.partials;
  args.max_blocks = max_blocks_per_seq;
  args.num_seqs = num_seqs;
  args.num_q_heads = num_q_heads;
  args.num_kv_heads = num_kv_heads;
  args.head_groups = geo.NHG;
  args.block_size = block_size;
  args.num_blocks = num_blocks;
  args.out_dtype = out_dtype;
  args.num_workers = geo.NW;
  args.num_q_tokens = num_q_tokens;
  args.causal = causal;
  args.lse = lse;
  // after_plan: a programmatic dependent launch right behind the plan kernel
  // that writes its plan, waiting for it before reading anything
  geo.overlap = overlap || after_plan;
  args.wait_first = after_plan ? 1 : 0;
  args.merge_by_caller = merge_by_caller ? 1 : 0;
  args.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  args.k_new = new_slots ? k_new : nullptr;
  args.v_new = new_slots ? v_new : nullptr;
  args.new_slots = new_slots;
  args.k_pool = const_cast<void*>(k_pool);
  args.v_pool = const_cast<void*>(v_pool);
  if (args_out) *args_out = args;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (kv_dtype == PKV_BF16) {
    switch (head_dim) {
      case 64: return run_bf16_64(geo, args, k_pool, v_pool, s);
      case 128: return run_bf16_128(geo, args, k_pool, v_pool, s);
      case 256: return run_bf16_256(geo, args, k_pool, v_pool, s);
    }
  } else {
    switch (head_dim) {
      case 64: return run_f32_64(geo, args, k_pool, v_pool, s);
      case 128: return run_f32_128(geo, args, k_pool, v_pool, s);
    }
  }
  return PKV_ERR_INVALID;
}

}  // namespace

int pkv_paged_decode_attn_run(const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* block_tables, int32_t max_blocks_per_seq,
                              const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                              int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                              int32_t out_dtype, void* workspace, size_t workspace_bytes,
                              pkv_stream_t stream) {
  return run_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                  num_kv_heads, head_dim, block_size, num_blocks, scale, kv_dtype, out, out_dtype,
                  workspace, workspace_bytes, stream, nullptr, nullptr, nullptr, 1, g_launch_overlap != 0);
}

int pkv_paged_decode_attn_append_run(const void* q, const void* k_new, const void* v_new,
                                     const int64_t* slot_mapping, void* k_pool, void* v_pool,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                     int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                                     int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                     pkv_stream_t stream) {
  if (num_seqs > 0 && !slot_mapping) return PKV_ERR_INVALID;
  return run_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                  num_kv_heads, head_dim, block_size, num_blocks, scale, kv_dtype, out, out_dtype,
                  workspace, workspace_bytes, stream, k_new, v_new, slot_mapping, 1, g_launch_overlap != 0);
}

int pkv_paged_decode_attn(const void* q, const void* k_pool, const void* v_pool,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                          int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                          int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                          int32_t out_dtype, void* workspace, size_t workspace_bytes,
                          pkv_stream_t stream) {
  Geometry geo;
  if (!geometry(num_seqs, num_q_heads, num_kv_heads, head_dim, kv_dtype, &geo)) return PKV_ERR_INVALID;
  int rc = check_common(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                        block_size, num_blocks, out, out_dtype, workspace, workspace_bytes, geo);
  if (rc != PKV_OK) return rc;
  if (!std::isfinite(scale)) return PKV_ERR_INVALID;
  if (num_seqs == 0) return PKV_OK;
  rc = do_plan(geo, seq_lens, workspace, static_cast<cudaStream_t>(stream));
  if (rc != PKV_OK) return rc;
  // the plan kernel just launched writes what the attention reads first: the
  // attention waits for it at its very top, its launch overlapping the plan's
  return run_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                  num_kv_heads, head_dim, block_size, num_blocks, scale, kv_dtype, out, out_dtype,
                  workspace, workspace_bytes, stream, nullptr, nullptr, nullptr, 1, false, 1, nullptr, true);
}

int pkv_paged_attn_multi_query(const void* q, int32_t num_q_tokens, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                               int32_t out_dtype, void* workspace, size_t workspace_bytes,
                               pkv_stream_t stream) {
  const int32_t hq_eff = multi_query_heads(num_q_tokens, num_q_heads, num_kv_heads);
  if (hq_eff <= 0) return PKV_ERR_INVALID;
  Geometry geo;
  if (!geometry(num_seqs, hq_eff, num_kv_heads, head_dim, kv_dtype, &geo)) return PKV_ERR_INVALID;
  int rc = check_common(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                        block_size, num_blocks, out, out_dtype, workspace, workspace_bytes, geo);
  if (rc != PKV_OK) return rc;
  if (!std::isfinite(scale)) return PKV_ERR_INVALID;
  if (num_seqs == 0) return PKV_OK;
  rc = do_plan(geo, seq_lens, workspace, static_cast<cudaStream_t>(stream));
  if (rc != PKV_OK) return rc;
  return run_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                  num_kv_heads, head_dim, block_size, num_blocks, scale, kv_dtype, out, out_dtype,
                  workspace, workspace_bytes, stream, nullptr, nullptr, nullptr, num_q_tokens, false, 1, nullptr,
                  true);
}

}  // extern "C"

// ===========================================================================
// Shared-prefix decode attention
// ===========================================================================
// Requests forked from one prompt share its full blocks (the same physical
// ids lead their block tables).  Decode attention over the whole history is
// split at the end of the shared part into two disjoint token ranges whose
// results combine exactly (the merge of online-softmax states):
//   prefix pass: per group, the members' queries are the columns of one
//     multi-token launch (no causal mask) over the shared blocks, so each
//     shared K/V tile is read once for the whole group; it writes o_p and
//     the log-sum-exp lse_p of every (member, head);
//   suffix pass: per request, plain decode over its own blocks after the
//     prefix (o_s, lse_s);
//   combine: out = (2^(lse_p - M) o_p + 2^(lse_s - M) o_s) / (2^(lse_p - M) +
//     2^(lse_s - M)), M = max(lse_p, lse_s); both empty gives 0.
// A gather kernel builds the grouped queries, the group and suffix tables and
// lengths in the workspace, and checks that members agree on the shared ids.
namespace {

struct CascadeLayout {
  size_t suf_ws = 0, pre_ws = 0, q_grp = 0, grp_table = 0, grp_len = 0, suf_table = 0, suf_len = 0;
  size_t o_p = 0, lse_p = 0, o_s = 0, lse_s = 0, total = 0;
  Geometry gs, gp;
  bool ok = false;
};

CascadeLayout cascade_layout(int32_t S, int32_t NG, int32_t T, int32_t Hq, int32_t Hkv, int32_t D, int32_t dtype,
                             int32_t max_blocks) {
  CascadeLayout c;
  const int32_t hq_eff = multi_query_heads(T, Hq, Hkv);
  if (S < 0 || NG < 0 || max_blocks < 0 || hq_eff <= 0) return c;
  if (!geometry(S, Hq, Hkv, D, dtype, &c.gs) || !geometry(NG, hq_eff, Hkv, D, dtype, &c.gp)) return c;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t es = dtype == PKV_BF16 ? 2 : 4;
  size_t o = 0;
  c.suf_ws = o;  o += up(c.gs.lay.total);        // first: its status word is the call's
  c.pre_ws = o;  o += up(c.gp.lay.total);
  c.q_grp = o;  o += up(es * size_t(NG) * T * Hq * D);
  c.grp_table = o;  o += up(4 * size_t(NG) * max_blocks);
  c.grp_len = o;  o += up(4 * size_t(NG));
  c.suf_table = o;  o += up(4 * size_t(S) * max_blocks);
  c.suf_len = o;  o += up(4 * size_t(S));
  c.o_p = o;  o += up(4 * size_t(NG) * T * Hq * D);
  c.lse_p = o;  o += up(4 * size_t(NG) * T * Hq);
  c.o_s = o;  o += up(4 * size_t(S) * Hq * D);
  c.lse_s = o;  o += up(4 * size_t(S) * Hq);
  c.total = o;
  c.ok = true;
  return c;
}

}  // namespace

namespace pkv {

struct PrepArgs {
  const char* q;
  const int32_t* tables;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t S;
  const int32_t* group_start;
  const int32_t* prefix_blocks;
  int32_t NG, T, row_bytes, B;
  char* q_grp;
  int32_t* grp_table;
  int32_t* grp_len;
  int32_t* suf_table;
  int32_t* suf_len;
  uint32_t* status;       // the call's status word (suffix workspace)
  uint32_t* pre_status;   // the shared-part pass's status word
  // the two plans
  int32_t Hq, Hkv, D, kv_dtype;
  int32_t s_NHG, s_NW;
  char* s_ws;
  size_t s_prefix, s_wplan, s_counters;
  int32_t g_Hq, g_NHG, g_NW;
  char* g_ws;
  size_t g_prefix, g_wplan, g_counters;
};

// The group of request s (the last g with group_start[g] <= s) and how many
// leading blocks s shares with it: prefix_blocks[g], or 0 when the claim is
// not valid for s (member index outside the group, group larger than T,
// block count out of range, or s shorter than the shared part).  The gather
// and both plans read the claim this one way.
// gs: group_start, or its copy in shared memory.
__device__ __forceinline__ int shared_blocks_of(const PrepArgs& p, const int32_t* gs, int s, int* g_out,
                                                int* i_out) {
  int lo = 0, hi = p.NG - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (gs[mid] <= s) lo = mid; else hi = mid - 1;
  }
  const int first = gs[lo], size = gs[lo + 1] - first;
  const int i = s - first;
  const int pb = p.prefix_blocks[lo];
  const bool bad = i < 0 || i >= size || size > p.T || pb < 0 || pb > p.max_blocks || p.seq_lens[s] < pb * p.B;
  *g_out = lo;
  *i_out = i;
  return bad ? -1 - pb : pb;  // < 0: not valid (the claim, encoded)
}

// One launch prepares both passes.  Blocks 0 .. S-1 gather request s: its row
// of the grouped queries and its own-part table (the group's first member
// also writes the group table and zeroes unused member rows).  Block S plans
// the own-part pass over the lengths seq_len - shared tokens, block S + 1 the
// shared-part pass over each group's shared tokens; they compute those
// lengths from the claims themselves, store them for the passes and plan
// from the stored values, so nothing in this launch waits for another block.
// Every block first copies group_start to shared memory (when it has at most
// kPrepSmemGroups groups): the group of a request is then a search in shared
// memory instead of a chain of dependent global loads.
constexpr int kPrepSmemGroups = 2048;

// Lengths the two plans see: a request's own tokens (its length minus the
// shared part), or a group's shared tokens (0 for an empty group).
struct CascadeLen {
  const PrepArgs* p;
  const int32_t* gs;  // group_start or its shared-memory copy
  bool group;
  __device__ int operator()(int x) const {
    int g, i;
    if (!group) {
      const int pb = shared_blocks_of(*p, gs, x, &g, &i);
      return p->seq_lens[x] - (pb > 0 ? pb : 0) * p->B;
    }
    const int first = gs[x];
    if (gs[x + 1] <= first) return 0;
    const int pb = shared_blocks_of(*p, gs, first, &g, &i);
    return (pb > 0 ? pb : 0) * p->B;
  }
};

__global__ void __launch_bounds__(kPlanThreads) cascade_prep_kernel(const PrepArgs p) {
  // The own-part pass behind this launch may be scheduled now: its CTAs
  // become resident while this launch runs and wait for it at their top.
  if (threadIdx.x == 0) grid_launch_dependents();
  __shared__ int32_t gs_sh[kPrepSmemGroups + 1];
  const bool gs_in_smem = p.NG <= kPrepSmemGroups;
  if (gs_in_smem)
    for (int g = threadIdx.x; g <= p.NG; g += blockDim.x) gs_sh[g] = p.group_start[g];
  __syncthreads();
  const int32_t* gs = gs_in_smem ? gs_sh : p.group_start;
  const int blk = blockIdx.x;
  if (blk >= p.S) {
    const bool group = blk == p.S + 1;
    const CascadeLen len{&p, gs, group};
    int32_t* lens = group ? p.grp_len : p.suf_len;
    const int n = group ? p.NG : p.S;
    // only the shared-part pass records into its status word, and it runs
    // after this launch: clear it here
    if (group && threadIdx.x == 0) *p.pre_status = 0u;
    for (int x = threadIdx.x; x < n; x += blockDim.x) lens[x] = len(x);
    __syncthreads();  // the plan reads the stored lengths (this block's writes)
    const auto stored = [lens](int x) { return lens[x]; };
    if (group) {
      plan_body(stored, p.NG, p.g_Hq, p.Hkv, p.g_NHG, p.D, p.kv_dtype, p.g_NW, p.g_ws, p.g_prefix, p.g_wplan,
                p.g_counters);
    } else {
      plan_body(stored, p.S, p.Hq, p.Hkv, p.s_NHG, p.D, p.kv_dtype, p.s_NW, p.s_ws, p.s_prefix, p.s_wplan,
                p.s_counters);
    }
    return;
  }
  const int s = blk;
  int g, i;
  const int pbc = shared_blocks_of(p, gs, s, &g, &i);
  if (pbc < 0) {
    if (threadIdx.x == 0) record_status(p.status, kStatusBadTable);
  }
  const int pbs = pbc < 0 ? 0 : pbc;
  const int first = gs[g], size = gs[g + 1] - first;
  const int mi = (i >= 0 && i < p.T) ? i : 0;
  // query row: q[s] -> q_grp[g][mi]
  const uint4* src = reinterpret_cast<const uint4*>(p.q + size_t(s) * p.row_bytes);
  uint4* dst = reinterpret_cast<uint4*>(p.q_grp + (size_t(g) * p.T + mi) * p.row_bytes);
  for (int u = threadIdx.x; u < p.row_bytes / 16; u += blockDim.x) dst[u] = src[u];
  const int32_t* row = p.tables + size_t(s) * p.max_blocks;
  const int32_t* lead = p.tables + size_t(first) * p.max_blocks;
  for (int j = threadIdx.x; j < p.max_blocks; j += blockDim.x) {
    p.suf_table[size_t(s) * p.max_blocks + j] = j + pbs < p.max_blocks ? row[j + pbs] : -1;
    if (j < pbs && row[j] != lead[j]) record_status(p.status, kStatusBadTable);  // not shared after all
  }
  if (i == 0) {
    for (int j = threadIdx.x; j < p.max_blocks; j += blockDim.x) p.grp_table[size_t(g) * p.max_blocks + j] = row[j];
    for (int m = size; m < p.T; ++m) {
      uint4* z = reinterpret_cast<uint4*>(p.q_grp + (size_t(g) * p.T + m) * p.row_bytes);
      for (int u = threadIdx.x; u < p.row_bytes / 16; u += blockDim.x) z[u] = make_uint4(0, 0, 0, 0);
    }
  }
}

// A lane's PER consecutive floats of a row (16-byte loads where they fit).
template <int PER>
__device__ __forceinline__ void load_row_slice(const float* __restrict__ src, float (&v)[PER]) {
#pragma unroll
  for (int i = 0; i < PER; i += (PER >= 4 ? 4 : 2)) {
    if constexpr (PER >= 4) {
      const float4 f = *reinterpret_cast<const float4*>(src + i);
      v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
    } else {
      const float2 f = *reinterpret_cast<const float2*>(src + i);
      v[i] = f.x; v[i + 1] = f.y;
    }
  }
}

// One warp per (request, query head): combine the two partial results.
// With 8 or 16 columns (GM) in the shared-part pass (merge_here), the pieces
// of its split pairs are merged here, column by column (merge_span, merge_pieces),
// instead of by a launch of their own; its whole pairs were written to
// o_p / lse_p.  Before waiting for the shared-part pass a warp finds its
// group and its pair's span (caller input and plan, written before that pass
// began); after it, one round trip loads the own part, the pieces' m and l
// and their o slices together.
// 128 threads and at most 72 registers (D <= 128): 28 warps per SM, so one
// warp per (request, query head) of a 256 x 16 batch is resident at once
// (with 96 registers the last third waited for a second wave, ~7 us).
constexpr int kCombineThreads = 128;
constexpr int kCombineSmemGroups = 4096;  // group_start kept in shared memory below this many groups
template <int D, int GM>
__global__ void __launch_bounds__(kCombineThreads, D <= 128 ? 7 : 4)
    cascade_combine_kernel(const DecodeArgs sp, int sp_check_hq, int sp_check_dtype, int merge_here,
                           const float* __restrict__ o_p, const float* __restrict__ lse_p,
                           const float* __restrict__ o_s, const float* __restrict__ lse_s,
                           const int32_t* __restrict__ group_start, int32_t NG, int32_t T, int32_t S,
                           int32_t Hq, int32_t Hkv, void* out, int32_t out_dtype, uint32_t* __restrict__ status,
                           const uint32_t* __restrict__ pre_status) {
  constexpr int PER = D / 32;  // output elements per lane
  // group_start is the caller's, and no launch of this call writes it: the
  // CTAs copy it to shared memory and find each warp's group while the
  // shared-part pass still runs (they are resident during its tail), instead
  // of a chain of dependent global loads after it.
  extern __shared__ int32_t gs_sh[];
  const bool gs_in_smem = NG < kCombineSmemGroups;
  if (gs_in_smem)
    for (int g = threadIdx.x; g <= NG; g += blockDim.x) gs_sh[g] = group_start[g];
  __syncthreads();
  const int32_t* gs = gs_in_smem ? gs_sh : group_start;
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool active = wid < static_cast<long long>(S) * Hq;
  int s = 0, h = 0, lo = 0, i = 0;
  MergeSpan span;
  bool split = false;
  if (active) {
    s = static_cast<int>(wid / Hq);
    h = static_cast<int>(wid % Hq);
    int hi = NG - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gs[mid] <= s) lo = mid; else hi = mid - 1;
    }
    i = s - gs[lo];
    i = i < 0 ? 0 : (i >= T ? T - 1 : i);
    // the shared-part pass's plan was written by the preparation launch
    if (merge_here) split = merge_span(sp, sp_check_hq, sp_check_dtype, D, lo, h / (Hq / Hkv), span);
  }
  // wait until the shared-part pass (and the own-part pass before it)
  // completed and their results are visible
  grid_dependency_wait();
  if (wid == 0 && lane == 0 && *pre_status) record_status(status, *pre_status);
  if (!active) return;
  const size_t pr = (static_cast<size_t>(lo) * T + i) * Hq + h;  // prefix row
  const size_t sr = static_cast<size_t>(s) * Hq + h;              // suffix row
  // the own part's loads are in flight with the shared part's
  const float ls = lse_s[sr];
  float os[PER];
  load_row_slice<PER>(o_s + sr * D + lane * PER, os);
  float op[PER], lp;
  if (split) {
    const int Gq = Hq / Hkv;
    float M, L, acc[PER];
    merge_pieces<D, GM, true>(sp, span, i * Gq + h % Gq, lane, M, L, acc);
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) op[e] = acc[e] * inv;
    lp = L > 0.f ? M + __log2f(L) : -INFINITY;
  } else {
    lp = lse_p[pr];
    load_row_slice<PER>(o_p + pr * D + lane * PER, op);
  }
  const float M = fmaxf(lp, ls);
  float wp = 0.f, wsf = 0.f;
  if (M != -INFINITY) {
    wp = exp2f(lp - M);
    wsf = exp2f(ls - M);
  }
  const float den = wp + wsf;
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const float v = (wp * op[e] + wsf * os[e]) * inv;
    store1(out, out_dtype, sr * D + lane * PER + e, v);
  }
}

}  // namespace pkv

extern "C" {

size_t pkv_shared_prefix_workspace_bytes(int32_t num_seqs, int32_t num_groups, int32_t max_group,
                                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t max_blocks_per_seq) {
  size_t best = 0;
  for (int dt : {PKV_BF16, PKV_F32}) {
    const CascadeLayout c = cascade_layout(num_seqs, num_groups, max_group, num_q_heads, num_kv_heads, head_dim,
                                           dt, max_blocks_per_seq);
    if (c.ok && c.total > best) best = c.total;
  }
  return best;
}

int pkv_paged_decode_attn_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* seq_lens, int32_t num_seqs, const int32_t* group_start,
                                        const int32_t* prefix_blocks, int32_t num_groups, int32_t max_group,
                                        int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                        int32_t block_size, int32_t num_blocks, float scale, int32_t kv_dtype,
                                        void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                        pkv_stream_t stream) {
  if (num_seqs < 0 || num_groups < 0 || (num_seqs > 0 && num_groups < 1) || num_groups > num_seqs ||
      max_group < 1 || max_group > 16)
    return PKV_ERR_INVALID;
  const CascadeLayout c = cascade_layout(num_seqs, num_groups, max_group, num_q_heads, num_kv_heads, head_dim,
                                         kv_dtype, max_blocks_per_seq);
  if (!c.ok) return PKV_ERR_INVALID;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < c.total) return PKV_ERR_INVALID;
  int rc = check_common(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, block_size,
                        num_blocks, out, out_dtype, workspace, c.gs.lay.total, c.gs);
  if (rc != PKV_OK) return rc;
  if (!std::isfinite(scale)) return PKV_ERR_INVALID;
  if (num_seqs == 0) return PKV_OK;
  if (!group_start || !prefix_blocks) return PKV_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(workspace);
  const int32_t row_bytes = num_q_heads * head_dim * (kv_dtype == PKV_BF16 ? 2 : 4);
  // The suffix workspace leads: its status word is the call's own; clear it
  // before anything of this call can record a fault.  The shared-part
  // pass's word is cleared by the preparation launch (the pass runs after
  // it); the combine folds it into the call's.
  cudaError_t e = cudaMemsetAsync(w + c.suf_ws, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return host::cuda_fail(e);
  PrepArgs pa{static_cast<const char*>(q), block_tables, max_blocks_per_seq, seq_lens, num_seqs, group_start,
              prefix_blocks, num_groups, max_group, row_bytes, block_size, w + c.q_grp,
              reinterpret_cast<int32_t*>(w + c.grp_table), reinterpret_cast<int32_t*>(w + c.grp_len),
              reinterpret_cast<int32_t*>(w + c.suf_table), reinterpret_cast<int32_t*>(w + c.suf_len),
              reinterpret_cast<uint32_t*>(w + c.suf_ws), reinterpret_cast<uint32_t*>(w + c.pre_ws),
              num_q_heads, num_kv_heads, head_dim, kv_dtype,
              c.gs.NHG, c.gs.NW, w + c.suf_ws, c.gs.lay.prefix, c.gs.lay.wplan, c.gs.lay.counters,
              c.gp.Hq, c.gp.NHG, c.gp.NW, w + c.pre_ws, c.gp.lay.prefix, c.gp.lay.wplan, c.gp.lay.counters};
  cascade_prep_kernel<<<num_seqs + 2, kPlanThreads, 0, st>>>(pa);
  rc = host::check_launch();
  if (rc != PKV_OK) return rc;
  // own-part pass: each request over its own blocks; a dependent launch whose
  // CTAs become resident during the preparation and wait for it at their top
  rc = run_impl(q, k_pool, v_pool, reinterpret_cast<const int32_t*>(w + c.suf_table), max_blocks_per_seq,
                reinterpret_cast<const int32_t*>(w + c.suf_len), num_seqs, num_q_heads, num_kv_heads, head_dim,
                block_size, num_blocks, scale, kv_dtype, w + c.o_s, PKV_F32, w + c.suf_ws, c.gs.lay.total,
                stream, nullptr, nullptr, nullptr, 1, false, 1, reinterpret_cast<float*>(w + c.lse_s),
                /*after_plan=*/true);
  if (rc != PKV_OK) return rc;
  DecodeArgs sp{};  // the shared-part pass's launch arguments, for the combine's merge
  // shared-part pass: groups x members, every member sees the whole shared
  // part.  It may start during the own-part pass's tail (launch overlap):
  // what it reads first -- its plan, the group tables and lengths, the pools
  // -- was written by the gather and plan kernels, which finished before
  // the own-part pass began; that pass writes only its own workspace and o_s.
  rc = run_impl(w + c.q_grp, k_pool, v_pool, reinterpret_cast<const int32_t*>(w + c.grp_table),
                max_blocks_per_seq, reinterpret_cast<const int32_t*>(w + c.grp_len), num_groups, num_q_heads,
                num_kv_heads, head_dim, block_size, num_blocks, scale, kv_dtype, w + c.o_p, PKV_F32,
                w + c.pre_ws, c.gp.lay.total, stream, nullptr, nullptr, nullptr, max_group, true, 0,
                reinterpret_cast<float*>(w + c.lse_p), false, /*merge_by_caller=*/true, &sp);
  if (rc != PKV_OK) return rc;
  const long long warps = static_cast<long long>(num_seqs) * num_q_heads;
  const int threads = kCombineThreads;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  // a programmatic dependent launch: its blocks are resident during the
  // shared-part pass's tail and start as soon as it completes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = num_groups < kCombineSmemGroups ? (num_groups + 1) * sizeof(int32_t) : 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // 8 or 16 columns in the shared-part pass (a general launch: it writes a
  // log-sum-exp): its split pairs are merged here
  const int merge_here = (c.gp.G == 16 || c.gp.G == 8) ? 1 : 0;
  const bool gm8 = c.gp.G == 8;
  auto combine = [&](auto kern) {
    return cudaLaunchKernelEx(&cfg, kern, sp, c.gp.Hq, kv_dtype, merge_here,
                              reinterpret_cast<const float*>(w + c.o_p), reinterpret_cast<const float*>(w + c.lse_p),
                              reinterpret_cast<const float*>(w + c.o_s), reinterpret_cast<const float*>(w + c.lse_s),
                              static_cast<const int32_t*>(group_start), num_groups, max_group, num_seqs,
                              num_q_heads, num_kv_heads, out, out_dtype, reinterpret_cast<uint32_t*>(w + c.suf_ws),
                              reinterpret_cast<const uint32_t*>(w + c.pre_ws));
  };
  switch (head_dim) {
    case 64: e = gm8 ? combine(cascade_combine_kernel<64, 8>) : combine(cascade_combine_kernel<64, 16>); break;
    case 128: e = gm8 ? combine(cascade_combine_kernel<128, 8>) : combine(cascade_combine_kernel<128, 16>); break;
    case 256: e = gm8 ? combine(cascade_combine_kernel<256, 8>) : combine(cascade_combine_kernel<256, 16>); break;
    default: return PKV_ERR_INVALID;
  }
  if (e != cudaSuccess) return host::cuda_fail(e);
  return host::check_launch();
}

int pkv_decode_status(void* workspace, pkv_stream_t stream) {
  if (!workspace) return PKV_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t st = 0;
  cudaError_t e = cudaMemcpyAsync(&st, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return host::cuda_fail(e);
  if (st) {
    const uint32_t zero = 0;
    e = cudaMemcpyAsync(workspace, &zero, sizeof(uint32_t), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return host::cuda_fail(e);
  }
  if (st & kStatusBadTable) return PKV_ERR_BAD_TABLE;
  if (st & kStatusTimeout) return PKV_ERR_DEVICE_TIMEOUT;
  if (st & kStatusPlanMismatch) return PKV_ERR_PLAN_MISMATCH;
  return PKV_OK;
}

}  // extern "C"

namespace pkv {

// One warp waits on an mbarrier that nothing arrives on, through the same
// bounded wait the decode kernel uses, and records the timeout.
__global__ void bounded_wait_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    pkv::mbar_init(pkv::smem_u32(&bar), 1);
    pkv::fence_mbar_init();
  }
  __syncwarp();
  if (!pkv::mbar_wait_bounded(pkv::smem_u32(&bar), 0, limit_ns) && threadIdx.x == 0)
    pkv::record_status(status, pkv::kStatusTimeout);
}

}  // namespace pkv

extern "C" {

int pkv_selftest_bounded_wait(unsigned long long limit_ns, void* workspace, size_t workspace_bytes,
                              pkv_stream_t stream) {
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < sizeof(WsHeader)) return PKV_ERR_INVALID;
  if (limit_ns == 0 || limit_ns > 100000000ull) return PKV_ERR_INVALID;  // at most 0.1 s
  pkv::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      &reinterpret_cast<WsHeader*>(workspace)->status, limit_ns);
  return host::check_launch();
}

int pkv_set_decode_kernel(int32_t which) {
  if (which < 0 || which > 2) return PKV_ERR_INVALID;
  g_kernel_choice = which;
  return PKV_OK;
}

int pkv_set_launch_overlap(int32_t on) {
  if (on != 0 && on != 1) return PKV_ERR_INVALID;
  g_launch_overlap = on;
  return PKV_OK;
}

}  // extern "C"

// ===========================================================================
// Allocation-free decode attention
// ===========================================================================
// Some callers cannot hand us device scratch: a plugin invoked by a host
// runtime that owns every device allocation and passes a kernel only its
// inputs and outputs, or a latency-critical serving loop that must never call
// cudaMalloc (it synchronises the device and can fail late under memory
// pressure).  For them the entry point below keeps its scratch in a
// fixed-size array that lives in this library's device image: every GPU that
// loads the library holds these bytes until the process exits, and no call
// allocates anything.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's name is only a host-side stand-in in host code: its device
// address is looked up with cudaGetSymbolAddress, with the device current,
// once per device context and cached.  The cache is keyed by the context's
// unique id, so after a cudaDeviceReset (a new context, the module loaded
// again, possibly at another address) the first call looks the address up
// again instead of using a stale one.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct NoAllocSlot {
  unsigned long long ctx_id = 0;  // 0: not set up
  void* ptr = nullptr;
};

std::mutex g_noalloc_mu;
NoAllocSlot g_noalloc[64];

bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return host::cuda_fail(e);
  if (dev < 0 || dev >= 64) return PKV_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  if (!have_id || g_noalloc[dev].ctx_id != id) {
    // set-up for this device context (also binds the context to the thread)
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return host::cuda_fail(e);
    if (!have_id && !current_context_id(&id)) id = 0;  // no id: look the address up on every call
    g_noalloc[dev].ctx_id = id;
    g_noalloc[dev].ptr = p;
    *out = p;
    return PKV_OK;
  }
  *out = g_noalloc[dev].ptr;
  return PKV_OK;
}

}  // namespace

extern "C" int pkv_paged_decode_attn_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                                             const int32_t* seq_lens, int32_t num_seqs,
                                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                             int32_t block_size, int32_t num_blocks, float scale,
                                             int32_t kv_dtype, void* out, int32_t out_dtype,
                                             pkv_stream_t stream) {
  Geometry geo;
  if (!geometry(num_seqs, num_q_heads, num_kv_heads, head_dim, kv_dtype, &geo)) return PKV_ERR_INVALID;
  // the limit is the documented one: the workspace size pkv_decode_workspace_bytes
  // states for the batch (the larger of the two storage types' layouts)
  if (pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim) > kNoAllocScratchBytes) {
    host::set_error("decode batch needs more scratch than the 16 MiB built into the library");
    return PKV_ERR_INVALID;
  }
  void* ws = nullptr;
  int rc = noalloc_scratch(&ws);
  if (rc != PKV_OK) return rc;
  // The array keeps the previous call's contents: clear the header (status
  // word and plan marker) before this call plans into it.
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(WsHeader), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return host::cuda_fail(e);
  return pkv_paged_decode_attn(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                               num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, kv_dtype,
                               out, out_dtype, ws, kNoAllocScratchBytes, stream);
}
