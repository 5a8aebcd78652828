// Cache-write kernels of libpkv: token append, copy-on-write block copy and
// slot mapping.
//
// "PagedAttention：让 KV cache 按需生长" (hs-black.github.io):
//   * slot of token t = block_table[t / B] * B + t % B, the pool row in the
//     [block][slot][kv head][dim] layout (sections "读 token 6，先查表，再找偏移"
//     and "把 token 6 变成真正的内存地址");
//   * append writes the new token's K and V into its slot, earlier blocks
//     never move (section "写满一块，再拿下一块");
//   * copy-on-write copies the valid prefix of a shared tail into a fresh block
//     of every layer before the write (sections "只读时共用，要写入时再分开" and
//     "一次写入，为什么会先少掉一个空闲块？"); stream order makes the copy visible
//     before the append that follows it (section "先确保分配成功，再改变可见状态").
//   * preemption by swap moves a request's blocks (every layer, K and V) to a
//     pinned host buffer and back, the alternative to recompute weighed in
//     section "腾出显存以后，还要付一次恢复成本".
// All four are pure data movement; each thread moves 16-byte vectors.
#include <cuda_runtime.h>

#include "../../include/pkv.h"
#include "pkv_host.h"

namespace {

constexpr int kMaxLayers = 128;

// One warp per (token, tensor): copy one token row (H_kv * D elements).
__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k,
                                                     const uint4* __restrict__ v,
                                                     const int64_t* __restrict__ slots, int n,
                                                     uint4* __restrict__ kp, uint4* __restrict__ vp,
                                                     int row_vec, long long total_slots) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= 2ll * n) return;
  const int tok = static_cast<int>(w >> 1);
  const bool is_v = (w & 1) != 0;
  const long long slot = slots[tok];
  if (slot < 0 || slot >= total_slots) return;
  const uint4* src = (is_v ? v : k) + static_cast<long long>(tok) * row_vec;
  uint4* dst = (is_v ? vp : kp) + slot * row_vec;
  for (int i = lane; i < row_vec; i += 32) dst[i] = src[i];
}

struct PoolPtrs {
  uint4* k[kMaxLayers];
  uint4* v[kMaxLayers];
};

// grid (copy, layer, tensor): copy the first n_valid slots of block src to dst.
__global__ void __launch_bounds__(256) block_copy_kernel(const __grid_constant__ PoolPtrs pools,
                                                         const int32_t* __restrict__ copies,
                                                         int row_vec, int B, int N) {
  const int c = blockIdx.x, layer = blockIdx.y, is_v = blockIdx.z;
  const int src = copies[3 * c + 0], dst = copies[3 * c + 1], nv = copies[3 * c + 2];
  if (src < 0 || src >= N || dst < 0 || dst >= N || src == dst || nv < 0 || nv > B) return;
  uint4* pool = is_v ? pools.v[layer] : pools.k[layer];
  const uint4* s = pool + static_cast<long long>(src) * B * row_vec;
  uint4* d = pool + static_cast<long long>(dst) * B * row_vec;
  const int n = nv * row_vec;
  for (int i = threadIdx.x; i < n; i += blockDim.x) d[i] = s[i];
}

// grid (block, layer, tensor): move one block of one layer's K or V between
// the pool and a host buffer laid out [n][layer][K,V][B * H_kv * d].
__global__ void __launch_bounds__(256) swap_kernel(const __grid_constant__ PoolPtrs pools,
                                                   const int32_t* __restrict__ blocks, int num_layers,
                                                   uint4* __restrict__ host, int block_vec, int N,
                                                   int to_host) {
  const int i = blockIdx.x, layer = blockIdx.y, is_v = blockIdx.z;
  const int b = blocks[i];
  if (b < 0 || b >= N) return;
  uint4* pool = (is_v ? pools.v[layer] : pools.k[layer]) + static_cast<long long>(b) * block_vec;
  uint4* h = host + ((static_cast<long long>(i) * num_layers + layer) * 2 + is_v) * block_vec;
  if (to_host) {
    for (int j = threadIdx.x; j < block_vec; j += blockDim.x) h[j] = pool[j];
  } else {
    for (int j = threadIdx.x; j < block_vec; j += blockDim.x) pool[j] = h[j];
  }
}

__global__ void slot_mapping_kernel(const int32_t* __restrict__ tables, int max_blocks,
                                    const int32_t* __restrict__ rows,
                                    const int32_t* __restrict__ positions, int n, int B,
                                    int64_t* __restrict__ slots) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int p = positions[i];
  if (p < 0) {
    slots[i] = -1;
    return;
  }
  const int r = rows ? rows[i] : i;
  if (p / B >= max_blocks) {
    slots[i] = -1;
    return;
  }
  const int32_t phys = tables[static_cast<long long>(r) * max_blocks + p / B];
  slots[i] = static_cast<int64_t>(phys) * B + p % B;
}

int esize(int dtype) { return dtype == PKV_BF16 ? 2 : (dtype == PKV_F32 ? 4 : 0); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool pow2_block(int B) { return B >= 1 && B <= 1024 && (B & (B - 1)) == 0; }

}  // namespace

extern "C" {

int pkv_kv_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t n_tokens,
                  void* k_pool, void* v_pool, int32_t num_kv_heads, int32_t head_dim,
                  int32_t block_size, int32_t num_blocks, int32_t dtype, pkv_stream_t stream) {
  const int es = esize(dtype);
  if (!es || n_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks < 0 ||
      !pow2_block(block_size))
    return PKV_ERR_INVALID;
  const long long row_bytes = static_cast<long long>(num_kv_heads) * head_dim * es;
  if (row_bytes % 16) return PKV_ERR_INVALID;
  if (n_tokens == 0) return PKV_OK;
  if (!k || !v || !slot_mapping || !k_pool || !v_pool) return PKV_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_pool) || !aligned16(v_pool)) return PKV_ERR_INVALID;
  const int row_vec = static_cast<int>(row_bytes / 16);
  const long long warps = 2ll * n_tokens;
  const long long blocks = (warps * 32 + 255) / 256;
  append_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, n_tokens,
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), row_vec,
      static_cast<long long>(num_blocks) * block_size);
  return host::check_launch();
}

int pkv_block_copy(void* const* k_pools, void* const* v_pools, int32_t num_layers,
                   const int32_t* copies, int32_t n_copies, int32_t num_kv_heads,
                   int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t dtype,
                   pkv_stream_t stream) {
  const int es = esize(dtype);
  if (!es || n_copies < 0 || num_layers < 1 || num_layers > kMaxLayers || num_kv_heads <= 0 ||
      head_dim <= 0 || num_blocks < 0 || !pow2_block(block_size))
    return PKV_ERR_INVALID;
  const long long row_bytes = static_cast<long long>(num_kv_heads) * head_dim * es;
  if (row_bytes % 16) return PKV_ERR_INVALID;
  if (n_copies == 0) return PKV_OK;
  if (!k_pools || !v_pools || !copies) return PKV_ERR_INVALID;
  PoolPtrs p{};
  for (int l = 0; l < num_layers; ++l) {
    if (!k_pools[l] || !v_pools[l] || !aligned16(k_pools[l]) || !aligned16(v_pools[l]))
      return PKV_ERR_INVALID;
    p.k[l] = static_cast<uint4*>(k_pools[l]);
    p.v[l] = static_cast<uint4*>(v_pools[l]);
  }
  dim3 grid(static_cast<unsigned>(n_copies), static_cast<unsigned>(num_layers), 2);
  block_copy_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      p, copies, static_cast<int>(row_bytes / 16), block_size, num_blocks);
  return host::check_launch();
}

int pkv_swap_blocks(void* const* k_pools, void* const* v_pools, int32_t num_layers,
                    const int32_t* blocks, int32_t n_blocks, void* host_buf, int32_t to_host,
                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                    int32_t dtype, pkv_stream_t stream) {
  const int es = esize(dtype);
  if (!es || n_blocks < 0 || num_layers < 1 || num_layers > kMaxLayers || num_kv_heads <= 0 ||
      head_dim <= 0 || num_blocks < 0 || !pow2_block(block_size) || (to_host != 0 && to_host != 1))
    return PKV_ERR_INVALID;
  const long long block_bytes = static_cast<long long>(block_size) * num_kv_heads * head_dim * es;
  if (block_bytes % 16) return PKV_ERR_INVALID;
  if (n_blocks == 0) return PKV_OK;
  if (!k_pools || !v_pools || !blocks || !host_buf || !aligned16(host_buf)) return PKV_ERR_INVALID;
  PoolPtrs p{};
  for (int l = 0; l < num_layers; ++l) {
    if (!k_pools[l] || !v_pools[l] || !aligned16(k_pools[l]) || !aligned16(v_pools[l]))
      return PKV_ERR_INVALID;
    p.k[l] = static_cast<uint4*>(k_pools[l]);
    p.v[l] = static_cast<uint4*>(v_pools[l]);
  }
  dim3 grid(static_cast<unsigned>(n_blocks), static_cast<unsigned>(num_layers), 2);
  swap_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      p, blocks, num_layers, static_cast<uint4*>(host_buf), static_cast<int>(block_bytes / 16), num_blocks,
      to_host);
  return host::check_launch();
}

int pkv_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* rows,
                     const int32_t* positions, int32_t n, int32_t block_size, int64_t* slots,
                     pkv_stream_t stream) {
  if (n < 0 || max_blocks_per_seq < 0 || block_size <= 0) return PKV_ERR_INVALID;
  if (n == 0) return PKV_OK;
  if (!block_tables || !positions || !slots) return PKV_ERR_INVALID;
  slot_mapping_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      block_tables, max_blocks_per_seq, rows, positions, n, block_size, slots);
  return host::check_launch();
}

}  // extern "C"
