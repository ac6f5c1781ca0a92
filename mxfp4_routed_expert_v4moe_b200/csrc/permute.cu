// Token permutation by expert: a deterministic, stable counting sort of the
// T*k (token, slot) pairs by expert id, which groups the rows each expert's
// GEMM consumes (the experts(flat, indices, weights) step of the MoE block,
// "Checked in its code" row "Shared expert").
//
// Small inputs (T*k <= kPermChunk): one CTA does histogram, scan and scatter.
// Large inputs: per-chunk histograms (one CTA per chunk of kPermChunk slots),
// one CTA scans experts and chunk bases, then one warp per chunk scatters its
// slots in order. Stability inside a chunk comes from walking the chunk in
// slot order, 32 slots at a time, with __match_any_sync ranking equal ids.
#include <mutex>
#include <unordered_map>

#include "launch.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

__device__ __forceinline__ bool id_ok(int e, int E) { return e >= 0 && e < E; }

// Exclusive scan of v over the block (blockDim.x == 1024, one value per
// thread); returns the exclusive prefix, *total gets the sum.
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_sums[lane] = wi - w;  // exclusive over warps
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - v;
  // total: last thread's inclusive value
  __shared__ int tot;
  if (threadIdx.x == blockDim.x - 1) tot = excl + v;
  __syncthreads();
  *total = tot;
  return excl;
}

__global__ void __launch_bounds__(1024) k_perm_single(int S, int E, const int32_t* __restrict__ ids,
                                                     int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                     int32_t* __restrict__ sorted_slot,
                                                     int32_t* __restrict__ slot_pos, uint32_t* status) {
  __shared__ int cnt[1024];
  __shared__ int cursor[1024];
  cnt[threadIdx.x] = 0;
  __syncthreads();
  bool bad = false;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const int e = ids[s];
    if (id_ok(e, E))
      atomicAdd(&cnt[e], 1);
    else
      bad = true;
  }
  if (bad) atomicOr(status, kStatusBadExpertId);
  __syncthreads();
  const int v = threadIdx.x < E ? cnt[threadIdx.x] : 0;
  int total;
  const int excl = block_exclusive_scan(v, &total);
  if (threadIdx.x < E) {
    counts[threadIdx.x] = v;
    offsets[threadIdx.x] = excl;
    cursor[threadIdx.x] = excl;
  }
  if (threadIdx.x == 0) offsets[E] = total;
  __syncthreads();
  if (threadIdx.x < 32) warp_stable_scatter(ids, 0, S, E, cursor, sorted_slot, slot_pos);
}

__global__ void __launch_bounds__(256) k_perm_hist(int S, int E, const int32_t* __restrict__ ids,
                                                   int32_t* __restrict__ chunk_counts, uint32_t* status) {
  __shared__ int cnt[1024];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int s0 = blockIdx.x * kPermChunk, s1 = min(S, s0 + kPermChunk);
  bool bad = false;
  for (int s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int e = ids[s];
    if (id_ok(e, E))
      atomicAdd(&cnt[e], 1);
    else
      bad = true;
  }
  if (bad) atomicOr(status, kStatusBadExpertId);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[size_t(blockIdx.x) * E + e] = cnt[e];
}

__global__ void __launch_bounds__(1024) k_perm_scan(int E, int nchunks, const int32_t* __restrict__ chunk_counts,
                                                    int32_t* __restrict__ chunk_base,
                                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  const int e = threadIdx.x;
  int tot = 0;
  if (e < E)
    for (int c = 0; c < nchunks; ++c) tot += chunk_counts[size_t(c) * E + e];
  int total;
  const int excl = block_exclusive_scan(e < E ? tot : 0, &total);
  if (e < E) {
    counts[e] = tot;
    offsets[e] = excl;
    int run = excl;
    for (int c = 0; c < nchunks; ++c) {
      chunk_base[size_t(c) * E + e] = run;
      run += chunk_counts[size_t(c) * E + e];
    }
  }
  if (threadIdx.x == 0) offsets[E] = total;
}

// One CTA per chunk, its 8 warps on consecutive sub-chunks of kPermChunk / 8
// slots: per-warp histograms give each warp its starting position per expert
// (the chunk's base plus the counts of the earlier sub-chunks), so the order
// stays the stable slot order.
constexpr int kScatterWarps = 8;
constexpr int kSubChunk = kPermChunk / kScatterWarps;

__global__ void __launch_bounds__(32 * kScatterWarps) k_perm_scatter(int S, int E, const int32_t* __restrict__ ids,
                                                                    const int32_t* __restrict__ chunk_base,
                                                                    int32_t* __restrict__ sorted_slot,
                                                                    int32_t* __restrict__ slot_pos) {
  extern __shared__ int pss[];  // [kScatterWarps][E] counts, then cursors
  const int warp = threadIdx.x >> 5;
  const int s0 = blockIdx.x * kPermChunk + warp * kSubChunk;
  const int s1 = min(S, s0 + kSubChunk);
  int* cnt = pss + warp * E;
  for (int e = threadIdx.x & 31; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  for (int s = s0 + (threadIdx.x & 31); s < s1; s += 32) {
    const int e = ids[s];
    if (id_ok(e, E)) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base[size_t(blockIdx.x) * E + e];
    for (int w = 0; w < kScatterWarps; ++w) {
      const int c = pss[w * E + e];
      pss[w * E + e] = run;  // becomes warp w's cursor
      run += c;
    }
  }
  __syncthreads();
  if (s0 < s1) warp_stable_scatter(ids, s0, s1, E, cnt, sorted_slot, slot_pos);
}

}  // namespace

cudaError_t launch_permute(const v4moe_config& c, int T, const int32_t* topk_ids, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos,
                           int32_t* chunk_counts, int32_t* chunk_base, int nchunks,
                           uint32_t* status, cudaStream_t st) {
  const int S = T * c.top_k;
  const int E = c.n_experts;
  if (S <= kPermChunk)
    return launch_kernel("perm_single", k_perm_single, dim3(1), dim3(1024), 0, st, false, S, E, topk_ids,
                         counts, offsets, sorted_slot, slot_pos, status);
  cudaError_t e = launch_kernel("perm_hist", k_perm_hist, dim3(nchunks), dim3(256), 0, st, false, S, E,
                                topk_ids, chunk_counts, status);
  if (e != cudaSuccess) return e;
  e = launch_kernel("perm_scan", k_perm_scan, dim3(1), dim3(1024), 0, st, false, E, nchunks,
                    (const int32_t*)chunk_counts, chunk_base, counts, offsets);
  if (e != cudaSuccess) return e;
  const size_t smem = size_t(kScatterWarps) * E * sizeof(int);
  set_smem(k_perm_scatter, smem);
  return launch_kernel("perm_scatter", k_perm_scatter, dim3(nchunks), dim3(32 * kScatterWarps), smem, st, false, S,
                       E, topk_ids, (const int32_t*)chunk_base, sorted_slot, slot_pos);
}

}  // namespace v4moe

// ---------------------------------------------------------------------------
// Permutation without a caller workspace.
//
// Some callers cannot hand the library a device buffer: runtimes whose device
// memory is planned once at start-up and may not grow afterwards, or host code
// that must not reach a device allocator (which may synchronise the device or
// fail under memory pressure). For them v4moe_permute_static keeps its scratch
// in the fixed array below, which every GPU that loads this library holds
// until the process exits.
namespace v4moe {
namespace {

constexpr int kStaticMaxSlots = 1 << 16;                          // T * top_k limit
constexpr int kStaticMaxChunks = kStaticMaxSlots / kPermChunk;    // 32
constexpr int kStaticStatusWords = 64;                            // 256-byte status block
constexpr size_t kStaticWords = kStaticStatusWords + size_t(2) * kStaticMaxChunks * 1024;

// Layout: [status block][chunk counts][chunk bases]. In host code this name
// only stands for the array; its device address comes from
// cudaGetSymbolAddress.
__device__ __align__(256) int32_t g_perm_scratch[kStaticWords];

std::mutex g_scratch_mu;
std::unordered_map<int, int32_t*> g_scratch_addr;  // device ordinal -> device address

// Device address of g_perm_scratch on the current device (looked up once per
// device, with that device current).
int32_t* static_scratch(cudaError_t* err) {
  int dev = -1;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  auto it = g_scratch_addr.find(dev);
  if (it != g_scratch_addr.end()) return it->second;
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_perm_scratch);
  if (*err != cudaSuccess) return nullptr;
  g_scratch_addr.emplace(dev, static_cast<int32_t*>(p));
  return static_cast<int32_t*>(p);
}

}  // namespace
}  // namespace v4moe

extern "C" int32_t v4moe_permute_static(const v4moe_config* cfg, int32_t T, const int32_t* topk_ids,
                                        int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                                        int32_t* slot_pos, void* stream) {
  using namespace v4moe;
  // The same argument rules as v4moe_permute, plus the fixed array's limit.
  if (!config_ok(cfg) || T < 0) return V4MOE_ERR_INVALID_ARG;
  if (!counts || !offsets) return V4MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !sorted_slot || !slot_pos)) return V4MOE_ERR_INVALID_ARG;
  if (int64_t(T) * cfg->top_k > kStaticMaxSlots) return V4MOE_ERR_INVALID_ARG;
  if (int32_t r = check_device()) return r;
  cudaError_t err = cudaSuccess;
  int32_t* base = static_scratch(&err);
  if (!base) {
    cudaGetLastError();
    return V4MOE_ERR_LAUNCH;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int S = T * cfg->top_k;
  const int nchunks = S > 0 ? (S + kPermChunk - 1) / kPermChunk : 1;
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  int32_t* chunk_counts = base + kStaticStatusWords;
  int32_t* chunk_base = chunk_counts + size_t(nchunks) * cfg->n_experts;
  // The status word is the only scratch that accumulates; start it at zero.
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) {
    cudaGetLastError();
    return V4MOE_ERR_LAUNCH;
  }
  const cudaError_t e = launch_permute(*cfg, T, topk_ids, counts, offsets, sorted_slot, slot_pos,
                                       chunk_counts, chunk_base, nchunks, status, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return V4MOE_ERR_LAUNCH;
  }
  return V4MOE_OK;
}
