// Decode attention entry points of libpkv: plan, partition (persistent
// warp-level stream-K over 16-token tiles) and merge kernels, plus the host
// side that validates arguments, builds the TMA tensor maps and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/pkv.h"
#include "pkv_decode_mma.cuh"
#include "pkv_host.h"

namespace pkv {

// ---------------------------------------------------------------------------
// Plan: tiles per request (prefix), and each worker's starting position.
// One CTA; work O(S + NW).
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ seq_lens,
                                                            int S, int Hq, int Hkv, int D,
                                                            int kv_dtype, int NW, char* ws,
                                                            size_t off_prefix, size_t off_wplan) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  int32_t* prefix = reinterpret_cast<int32_t*>(ws + off_prefix);
  int4* wplan = reinterpret_cast<int4*>(ws + off_wplan);
  __shared__ long long warp_tot[kPlanThreads / 32];
  __shared__ long long total_sh;

  const int tid = threadIdx.x;
  const int chunk = (S + kPlanThreads - 1) / kPlanThreads;
  const int s0 = min(S, tid * chunk), s1 = min(S, s0 + chunk);
  long long local = 0;
  for (int s = s0; s < s1; ++s) local += ntiles_of(seq_lens[s]);
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
    long long w = warp_tot[lane];
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) total_sh = wi;
  }
  __syncthreads();
  long long run = warp_tot[warp] + incl - local;
  for (int s = s0; s < s1; ++s) {
    prefix[s] = static_cast<int32_t>(run);
    run += ntiles_of(seq_lens[s]);
  }
  const long long total_seq_tiles = total_sh;
  if (tid == 0) prefix[S] = static_cast<int32_t>(total_seq_tiles);
  const long long T = total_seq_tiles * Hkv;

  // Worker starts: worker v begins at tile a_v = floor(v T / NW).  Each
  // request's thread writes the workers whose start falls in its tile range.
  if (T == 0) {
    for (int v = tid; v < NW; v += kPlanThreads) wplan[v] = make_int4(0, 0, 0, 0);
  } else {
    long long start = (warp_tot[warp] + incl - local) * Hkv;
    for (int s = s0; s < s1; ++s) {
      const long long nt = ntiles_of(seq_lens[s]);
      const long long end = start + nt * Hkv;
      if (nt > 0) {
        long long v = (start * NW + T - 1) / T;
        for (; v < NW; ++v) {
          const long long a = range_begin(static_cast<int>(v), T, NW);
          if (a >= end) break;
          const long long b = range_begin(static_cast<int>(v) + 1, T, NW);
          wplan[v] = make_int4(static_cast<int>(a), static_cast<int>(b), s, static_cast<int>(a - start));
        }
      }
      start = end;
    }
  }
  if (tid == 0) {
    hdr->num_seqs = S;
    hdr->num_q_heads = Hq;
    hdr->num_kv_heads = Hkv;
    hdr->head_dim = D;
    hdr->kv_dtype = kv_dtype;
    hdr->num_workers = NW;
    hdr->total_tiles = T;
    hdr->planned = 1;
  }
}

// ---------------------------------------------------------------------------
// Partition: persistent grid, one stream-K worker per warp.
// ---------------------------------------------------------------------------
template <class Core, int W, int DEPTH>
struct Smem {
  static constexpr int kStages = DEPTH * Core::kStageBytes;
  static constexpr int kScratch = Core::kScratchBytes;
  static constexpr int kMeta = DEPTH * int(sizeof(StageMeta));
  static constexpr int kBatchInts = kBatch * (4 + kMaxBoxes);
  static constexpr int kBatchB = kBatchInts * 4;
  static constexpr int kBars = DEPTH * 8;
  static constexpr int kPerWarp =
      round_up(kStages + kScratch + kMeta + kBatchB + kBars, Core::kAlign);
  static constexpr int kTotal = W * kPerWarp + Core::kAlign;  // + slack to align the base
};

struct TmaMaps {
  CUtensorMap k;
  CUtensorMap v;
};

template <class Core, int G, int W, int DEPTH>
__global__ void __launch_bounds__(W * 32, 1)
    partition_kernel(const __grid_constant__ TmaMaps maps, const DecodeArgs a, int check_S,
                     int check_Hq, int check_Hkv, int check_D, int check_dtype) {
  using SM = Smem<Core, W, DEPTH>;
  extern __shared__ char smem_raw[];
  char* base = reinterpret_cast<char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + Core::kAlign - 1) & ~uintptr_t(Core::kAlign - 1));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  char* wbase = base + warp * SM::kPerWarp;
  char* stages = wbase;
  float* scratch = reinterpret_cast<float*>(wbase + SM::kStages);
  StageMeta* meta = reinterpret_cast<StageMeta*>(wbase + SM::kStages + SM::kScratch);
  int32_t* bt = reinterpret_cast<int32_t*>(wbase + SM::kStages + SM::kScratch + SM::kMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(wbase + SM::kStages + SM::kScratch + SM::kMeta + SM::kBatchB);

  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  uint32_t* status = &hdr->status;
  if (hdr->planned != 1 || hdr->num_seqs != check_S || hdr->num_q_heads != check_Hq ||
      hdr->num_kv_heads != check_Hkv || hdr->head_dim != check_D || hdr->kv_dtype != check_dtype ||
      hdr->num_workers != a.num_workers) {
    if (threadIdx.x == 0) record_status(status, kStatusPlanMismatch);
    return;
  }
  const int v = blockIdx.x * W + warp;  // this warp's worker id
  const int4 wp = reinterpret_cast<const int4*>(a.ws + a.off_wplan)[v];
  const int ntiles = wp.y - wp.x;
  if (ntiles <= 0) return;

  const int S = a.num_seqs, Hkv = a.num_kv_heads, Bsz = a.block_size;
  const int Hq = a.num_q_heads;
  const int box_rows = Bsz < kTile ? Bsz : kTile;
  const int nbox = kTile / box_rows;  // boxes per tile per chunk
  const uint64_t pol = policy_evict_first();

  if (lane == 0) {
    for (int i = 0; i < DEPTH; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  // Lookahead cursor (warp-uniform): request cs, offset coff within its
  // Hkv * nt(cs) tiles.
  int cs = wp.z, coff = wp.w;
  int last_s = -1, last_g = -1;

  auto compute_batch = [&](int kb) {
    if (kb + lane < ntiles) {
      int s = cs, off = coff + lane;
      int len = a.seq_lens[s];
      int nt = ntiles_of(len);
      while (off >= Hkv * nt) {
        off -= Hkv * nt;
        if (s + 1 >= S) {  // inconsistent with the plan: stop here
          record_status(status, kStatusPlanMismatch);
          off = 0;
          break;
        }
        ++s;
        len = a.seq_lens[s];
        nt = ntiles_of(len);
      }
      const int g = nt > 0 ? off / nt : 0;
      const int j = nt > 0 ? off % nt : 0;
      const int nvalid = min(kTile, len - j * kTile);
      const int nblk = (len + Bsz - 1) / Bsz;
      const int lb0 = (j * kTile) / Bsz;
      int32_t* e = bt + lane * (4 + kMaxBoxes);
      e[0] = s;
      e[1] = g;
      e[2] = j;
      e[3] = (nvalid << 8) | (j == nt - 1 ? 2 : 0);
      const int32_t* row = a.block_tables + static_cast<size_t>(s) * a.max_blocks;
#pragma unroll
      for (int b = 0; b < kMaxBoxes; ++b) {
        int phys = -1;
        if (b < nbox && lb0 + b < nblk) {
          if (lb0 + b >= a.max_blocks) {  // length beyond the table row: caller error
            record_status(status, kStatusBadTable);
            e[4 + b] = -1;
            continue;
          }
          phys = row[lb0 + b];
          if (phys < 0 || phys >= a.num_blocks) {
            record_status(status, kStatusBadTable);
            phys = a.num_blocks;  // out of the tensor map: TMA fills zeros
          }
        }
        e[4 + b] = phys;
      }
      // carry the cursor: the last lane's position, one tile further
      cs = s;
      coff = off + 1;
    }
    // the cursor for the next batch comes from lane 31
    cs = __shfl_sync(0xffffffffu, cs, 31);
    coff = __shfl_sync(0xffffffffu, coff, 31);
    __syncwarp();
  };

  auto issue = [&](int k) {
    if ((k % kBatch) == 0) compute_batch(k);
    if (lane == 0) {
      const int32_t* e = bt + (k % kBatch) * (4 + kMaxBoxes);
      const int s = e[0], g = e[1], j = e[2];
      const bool newpair = (s != last_s) || (g != last_g);
      last_s = s;
      last_g = g;
      const int st = k % DEPTH;
      char* stage = stages + st * Core::kStageBytes;
      meta[st].s = s;
      meta[st].g = g;
      meta[st].j = j;
      meta[st].flags = e[3] | (newpair ? 1 : 0);
      const uint32_t bar = smem_u32(&bars[st]);
      int nb = 0;
#pragma unroll
      for (int b = 0; b < kMaxBoxes; ++b) nb += (b < nbox && e[4 + b] >= 0) ? 1 : 0;
      const uint32_t box_bytes = static_cast<uint32_t>(box_rows * Core::kChunkRowBytes);
      uint32_t bytes = 2u * nb * Core::kChunks * box_bytes;
      if (newpair) bytes += Core::QB;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bar, bytes);
      if (newpair) {
        const char* qsrc = reinterpret_cast<const char*>(a.q) +
                           (static_cast<size_t>(s) * Hq + static_cast<size_t>(g) * G) * Core::ROWB;
        bulk_load(smem_u32(stage + Core::kQOff), qsrc, Core::QB, bar);
      }
      const int slot0 = Bsz >= kTile ? (j * kTile) % Bsz : 0;
#pragma unroll
      for (int b = 0; b < kMaxBoxes; ++b) {
        const int phys = e[4 + b];
        if (b < nbox && phys >= 0) {
#pragma unroll
          for (int c = 0; c < Core::kChunks; ++c) {
            const uint32_t off = c * Core::kChunkBytes + b * box_bytes;
            tma_load_4d(smem_u32(stage + Core::kKOff + off), &maps.k, c * Core::kBoxInner, slot0, g,
                        phys, bar, pol);
            tma_load_4d(smem_u32(stage + Core::kVOff + off), &maps.v, c * Core::kBoxInner, slot0, g,
                        phys, bar, pol);
          }
        }
      }
    }
    __syncwarp();
  };

  const int prologue = ntiles < DEPTH ? ntiles : DEPTH;
  for (int k = 0; k < prologue; ++k) issue(k);

  typename Core::State state;
  bool have = false;
  int ps = 0, pg = 0, jfirst = 0;
  bool last_is_end = false;
  float* partials = reinterpret_cast<float*>(a.ws + a.off_partials);
  constexpr int PS = part_stride(G, Core::ROWB / Core::ESZ);
  constexpr int D = Core::ROWB / Core::ESZ;

  auto flush = [&]() {
    const bool complete = (jfirst == 0) && last_is_end;
    const size_t out_row = (static_cast<size_t>(ps) * Hq + static_cast<size_t>(pg) * G) * D;
    float* part = partials + static_cast<size_t>(v + ps * Hkv + pg) * PS;
    Core::finish(state, complete, a.out, a.out_dtype, out_row, part, lane);
  };

  for (int k = 0; k < ntiles; ++k) {
    const int st = k % DEPTH;
    if (!mbar_wait_bounded(smem_u32(&bars[st]), (k / DEPTH) & 1)) {
      if (lane == 0) record_status(status, kStatusTimeout);
      return;
    }
    const StageMeta m = meta[st];
    const char* stage = stages + st * Core::kStageBytes;
    if (m.flags & 1) {
      if (have) flush();
      have = true;
      ps = m.s;
      pg = m.g;
      jfirst = m.j;
      Core::begin_pair(state, stage + Core::kQOff, a.scale_log2, lane);
    }
    const int nvalid = m.flags >> 8;
    last_is_end = (m.flags & 2) != 0;
    if constexpr (Core::kSwizzle) {
      Core::tile(state, stage + Core::kKOff, stage + Core::kVOff, nvalid, a.scale_log2, lane);
    } else {
      Core::tile(state, stage + Core::kKOff, stage + Core::kVOff, nvalid, scratch, lane);
    }
    __syncwarp();
    if (k + DEPTH < ntiles) issue(k + DEPTH);
  }
  if (have) flush();
}

// ---------------------------------------------------------------------------
// Merge: one warp per (request, KV head) pair whose tiles span several
// workers; combines their partial states with the same rescaling rule.
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(256) merge_kernel(const DecodeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.num_kv_heads, Hq = a.num_q_heads;
  const long long p = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (p >= static_cast<long long>(a.num_seqs) * Hkv) return;
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
  if (hdr->planned != 1) return;
  const int s = static_cast<int>(p / Hkv), g = static_cast<int>(p % Hkv);
  const int len = a.seq_lens[s];
  constexpr int PER = D / 32;  // output elements per lane
  const size_t out_row = (static_cast<size_t>(s) * Hq + static_cast<size_t>(g) * G) * D;
  if (len <= 0) {
    for (int k = 0; k < G; ++k)
      for (int i = 0; i < PER; ++i) store1(a.out, a.out_dtype, out_row + k * D + lane * PER + i, 0.f);
    return;
  }
  const int32_t* prefix = reinterpret_cast<const int32_t*>(a.ws + a.off_prefix);
  const long long T = hdr->total_tiles;
  const int NW = a.num_workers;
  const long long nt = ntiles_of(len);
  const long long start = static_cast<long long>(prefix[s]) * Hkv + g * nt;
  const int v0 = owner_of(start, T, NW), v1 = owner_of(start + nt - 1, T, NW);
  if (v0 == v1) return;  // the single worker wrote the output itself
  constexpr int PS = part_stride(G, D);
  const float* partials = reinterpret_cast<const float*>(a.ws + a.off_partials);
  for (int k = 0; k < G; ++k) {
    float M = -INFINITY;
    for (int v = v0; v <= v1; ++v) {
      if (range_begin(v, T, NW) == range_begin(v + 1, T, NW)) continue;
      M = fmaxf(M, partials[static_cast<size_t>(v + p) * PS + G * D + k]);
    }
    float L = 0.f;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    for (int v = v0; v <= v1; ++v) {
      if (range_begin(v, T, NW) == range_begin(v + 1, T, NW)) continue;
      const float* part = partials + static_cast<size_t>(v + p) * PS;
      const float w = exp2f(part[G * D + k] - M);
      L = fmaf(w, part[G * D + G + k], L);
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, part[k * D + lane * PER + i], acc[i]);
    }
    const float inv = 1.f / L;
#pragma unroll
    for (int i = 0; i < PER; ++i) store1(a.out, a.out_dtype, out_row + k * D + lane * PER + i, acc[i] * inv);
  }
}

}  // namespace pkv

// ===========================================================================
// Host side
// ===========================================================================
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

int g_kernel_choice = 0;  // 0 auto, 1 fma, 2 mma

bool valid_dtype(int d) { return d == PKV_BF16 || d == PKV_F32; }
int esize(int d) { return d == PKV_BF16 ? 2 : 4; }

bool shape_ok(int Hq, int Hkv, int D, int dtype) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return false;
  if (dtype == PKV_BF16) return D == 64 || D == 128 || D == 256;
  if (dtype == PKV_F32) return D == 64 || D == 128;
  return false;
}

// Warps per SM that act as workers; the plan and every kernel variant agree.
int workers_per_sm(int D, int dtype) { return D * esize(dtype) >= 512 ? 4 : 8; }

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

// Pool viewed as 4-D (d, slot, kv head, block), box (inner, rows, 1, 1).
bool make_pool_map(CUtensorMap* m, const void* pool, int dtype, int D, int B, int Hkv, int N,
                   int box_inner, int box_rows, bool swizzle) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = static_cast<cuuint64_t>(esize(dtype));
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

struct Geometry {
  int S, Hq, Hkv, G, D, dtype, NW;
  WsLayout lay;
};

bool geometry(int S, int Hq, int Hkv, int D, int dtype, Geometry* g) {
  if (S < 0 || !valid_dtype(dtype) || !shape_ok(Hq, Hkv, D, dtype)) return false;
  const int sms = num_sms_current();
  if (sms <= 0) return false;
  const int NW = sms * workers_per_sm(D, dtype);
  *g = Geometry{S, Hq, Hkv, Hq / Hkv, D, dtype, NW, WsLayout(S, Hkv, Hq / Hkv, D, NW)};
  return true;
}

template <class Core, int G, int W, int DEPTH>
int launch_partition(const Geometry& geo, const DecodeArgs& args, const void* k_pool, const void* v_pool,
                     cudaStream_t stream) {
  using SM = Smem<Core, W, DEPTH>;
  static_assert(SM::kTotal <= 227 * 1024, "shared memory budget");
  TmaMaps maps;
  const int box_rows = args.block_size < kTile ? args.block_size : kTile;
  if (!make_pool_map(&maps.k, k_pool, geo.dtype, geo.D, args.block_size, geo.Hkv, args.num_blocks,
                     Core::kBoxInner, box_rows, Core::kSwizzle) ||
      !make_pool_map(&maps.v, v_pool, geo.dtype, geo.D, args.block_size, geo.Hkv, args.num_blocks,
                     Core::kBoxInner, box_rows, Core::kSwizzle)) {
    host::set_error("cuTensorMapEncodeTiled failed");
    return PKV_ERR_CUDA;
  }
  auto kern = partition_kernel<Core, G, W, DEPTH>;
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal);
    if (e != cudaSuccess) return host::cuda_fail(e);
    configured_dev = dev;
  }
  const int grid = geo.NW / W;
  kern<<<grid, W * 32, SM::kTotal, stream>>>(maps, args, geo.S, geo.Hq, geo.Hkv, geo.D, geo.dtype);
  return host::check_launch();
}

template <class Core, int G>
int launch_core(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
                cudaStream_t stream) {
  constexpr int W = (Core::ROWB >= 512) ? 4 : 8;
  constexpr int fixed = Core::kScratchBytes + kBatch * (4 + kMaxBoxes) * 4 + 64;
  constexpr int per_warp = (220 * 1024) / W - Core::kAlign;
  constexpr int depth_raw = (per_warp - fixed) / Core::kStageBytes;
  constexpr int DEPTH = depth_raw > 4 ? 4 : (depth_raw < 2 ? 2 : depth_raw);
  return launch_partition<Core, G, W, DEPTH>(geo, args, k, v, stream);
}

template <int D, int G>
int launch_merge(const Geometry& geo, const DecodeArgs& args, cudaStream_t stream) {
  const long long pairs = static_cast<long long>(geo.S) * geo.Hkv;
  if (pairs == 0) return PKV_OK;
  const long long blocks = (pairs + 7) / 8;
  merge_kernel<D, G><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(args);
  return host::check_launch();
}

template <int D, int G>
int run_dg(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
           cudaStream_t stream) {
  int rc;
  if (geo.dtype == PKV_F32) {
    if constexpr (D <= 128) {
      rc = launch_core<FmaCore<float, D, G>, G>(geo, args, k, v, stream);
    } else {
      return PKV_ERR_INVALID;
    }
  } else {
    bool use_mma = false;
    if constexpr (G <= 8) use_mma = args.block_size >= 8 && g_kernel_choice != 1;
    if (use_mma) {
      if constexpr (G <= 8) rc = launch_core<MmaCore<D, G>, G>(geo, args, k, v, stream);
      else rc = PKV_ERR_INVALID;
    } else {
      rc = launch_core<FmaCore<__nv_bfloat16, D, G>, G>(geo, args, k, v, stream);
    }
  }
  if (rc != PKV_OK) return rc;
  return launch_merge<D, G>(geo, args, stream);
}

template <int D>
int run_d(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v, cudaStream_t s) {
  switch (geo.G) {
    case 1: return run_dg<D, 1>(geo, args, k, v, s);
    case 2: return run_dg<D, 2>(geo, args, k, v, s);
    case 4: return run_dg<D, 4>(geo, args, k, v, s);
    case 8: return run_dg<D, 8>(geo, args, k, v, s);
    case 16: return run_dg<D, 16>(geo, args, k, v, s);
  }
  return PKV_ERR_INVALID;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int do_plan(const Geometry& geo, const int32_t* seq_lens, void* ws, cudaStream_t stream) {
  plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, geo.S, geo.Hq, geo.Hkv, geo.D, geo.dtype,
                                              geo.NW, static_cast<char*>(ws), geo.lay.prefix,
                                              geo.lay.wplan);
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
  // flattened tile indices are int32
  const long long max_tiles_seq = (static_cast<long long>(max_blocks) * B + kTile - 1) / kTile;
  if (static_cast<long long>(S) * geo.Hkv * max_tiles_seq >= (1ll << 31)) return PKV_ERR_INVALID;
  return PKV_OK;
}

}  // namespace

extern "C" {

size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim) {
  Geometry g;
  // the layout does not depend on the storage type beyond the worker count;
  // size for the larger of the two.
  size_t best = 0;
  for (int dt : {PKV_BF16, PKV_F32}) {
    if (geometry(num_seqs, num_q_heads, num_kv_heads, head_dim, dt, &g) && g.lay.total > best)
      best = g.lay.total;
  }
  return best;
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

int pkv_paged_decode_attn_run(const void* q, const void* k_pool, const void* v_pool,
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
  DecodeArgs args{};
  args.q = q;
  args.block_tables = block_tables;
  args.seq_lens = seq_lens;
  args.out = out;
  args.ws = static_cast<char*>(workspace);
  args.off_prefix = geo.lay.prefix;
  args.off_wplan = geo.lay.wplan;
  args.off_partials = geo.lay.partials;
  args.max_blocks = max_blocks_per_seq;
  args.num_seqs = num_seqs;
  args.num_q_heads = num_q_heads;
  args.num_kv_heads = num_kv_heads;
  args.block_size = block_size;
  args.num_blocks = num_blocks;
  args.out_dtype = out_dtype;
  args.num_workers = geo.NW;
  args.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (head_dim) {
    case 64: return run_d<64>(geo, args, k_pool, v_pool, s);
    case 128: return run_d<128>(geo, args, k_pool, v_pool, s);
    case 256: return run_d<256>(geo, args, k_pool, v_pool, s);
  }
  return PKV_ERR_INVALID;
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
  return pkv_paged_decode_attn_run(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens,
                                   num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                   num_blocks, scale, kv_dtype, out, out_dtype, workspace,
                                   workspace_bytes, stream);
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

int pkv_set_decode_kernel(int32_t which) {
  if (which < 0 || which > 2) return PKV_ERR_INVALID;
  g_kernel_choice = which;
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

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device.  The array's
// name is only a host-side stand-in in host code, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return host::cuda_fail(e);
  if (dev < 0 || dev >= 64) return PKV_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return host::cuda_fail(e);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
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
  if (geo.lay.total > kNoAllocScratchBytes) {
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
