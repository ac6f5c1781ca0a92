// Router of the DeepSeek-V4-Flash MoE layer on tcgen05 ("Checked in its code"
// rows "Mixture of experts" and "Auxiliary-loss-free load balancing
// (selection bias)"; "config.json" scoring_func sqrtsoftplus, topk_method
// noaux_tc, norm_topk_prob, routed_scaling_factor; hash layers per
// "DeepSeek-V4-Flash export design", section "Source configuration").
//
//  * k_route_gemm: logits x . gate^T as a bf16 tcgen05 GEMM (exact products,
//    fp32 accumulation in TMEM), TMA on both operands: tile = 128 tokens (M)
//    x up to 256 experts (N), the reduction split into ksplit parts so that
//    at least a full wave of CTAs runs. Each CTA writes its partial logits.
//  * k_route_select: one warp per token sums the partial logits in split
//    order (deterministic), takes sqrt(softplus), and selects: the k largest
//    s + bias (ties to the lower id, ids ascending; weights from the unbiased
//    s, normalised, x routed_scaling_factor), or the token's tid2eid row.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int RT = 128;  // tokens per tile (MMA M)
constexpr int RN = 256;  // experts per tile (largest MMA N)
constexpr int RK = 64;   // K per stage: 64 bf16 = one 128-byte swizzle atom
constexpr int kRStages = 4;
constexpr int kRThreads = 192;  // warp 0 TMA, warp 1 MMA and TMEM, warps 2-5 epilogue
constexpr int kRA = RT * RK * 2;
constexpr uint32_t kRTries = 1u << 21;

struct RBars {
  uint64_t full[kRStages];
  uint64_t empty[kRStages];
  uint64_t acc;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool rwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  for (uint32_t i = 0; i < kRTries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
  return false;
}

// grid (token tiles, K splits, expert tiles); box_n: gate rows per TMA box.
__global__ void __launch_bounds__(kRThreads, 1)
    k_route_gemm(int T, int E, int nk, int nk_per, int box_n, float* __restrict__ part, uint32_t* status,
                 const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage = kRA + box_n * RK * 2;
  RBars& B = *reinterpret_cast<RBars*>(smem + kRStages * stage);
  volatile int* abort_flag = &B.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * RT, ks = blockIdx.y, e0 = blockIdx.z * box_n;
  const int c0 = ks * nk_per, c1 = min(nk, c0 + nk_per);
  const int ne = min(box_n, E - e0);        // experts of this tile
  const int n_mma = (ne + 15) / 16 * 16;    // MMA N (columns past ne read zero rows)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&B.full[s], 1);
      mbar_init(&B.empty[s], 1);
    }
    mbar_init(&B.acc, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&B.tmem_base, RN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;
  pdl_wait();  // x may come from an earlier kernel

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmG);
    int issued = 0;
    for (int c = c0; c < c1; ++c, ++issued) {
      const int s = issued % kRStages;
      const uint32_t u = issued / kRStages;
      if (!rwait(&B.empty[s], (u & 1u) ^ 1u, abort_flag, status)) break;
      char* st = smem + s * stage;
      mbar_arrive_expect_tx(&B.full[s], uint32_t(stage));
      tma_load_2d(st, &tmX, c * RK, t0, &B.full[s]);
      tma_load_2d(st + kRA, &tmG, c * RK, e0, &B.full[s]);
    }
    // nothing may still be landing in shared memory when the CTA exits
    for (int q = 0; q < kRStages && q < issued; ++q) {
      const int gq = issued - 1 - q;
      mbar_wait_bounded(&B.full[gq % kRStages], uint32_t(gq / kRStages) & 1u, kRTries);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16_f32(RT, n_mma);
    int done = 0;
    for (int c = c0; c < c1; ++c, ++done) {
      const int s = done % kRStages;
      if (!rwait(&B.full[s], uint32_t(done / kRStages) & 1u, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * stage), b0 = a0 + kRA;
#pragma unroll
      for (int kk = 0; kk < RK / 16; ++kk)
        umma_f16_ss(tmem, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                    (c > c0 || kk > 0) ? 1u : 0u);
      umma_commit(&B.empty[s]);
    }
    umma_commit(&B.acc);
  } else if (warp >= 2) {
    // epilogue: thread = token (TMEM lane), columns = experts of the tile
    const int q = warp & 3;
    const int t = t0 + 32 * q + lane;
    if (rwait(&B.acc, 0, abort_flag, status) && c1 > c0) {
      tc_fence_after();
      for (int cc = 0; cc < n_mma; cc += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t(32 * q) << 16) + cc, r);
        tmem_wait_ld();
        if (t < T) {
          float* dst = part + (size_t(ks) * T + t) * E + e0 + cc;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (cc + i < ne) dst[i] = __uint_as_float(r[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, RN);
  }
}

// One warp per token: logits = sum of the splits' partials in split order,
// s = sqrt(softplus(logit)) in shared memory, then the selection.
template <bool HASH>
__global__ void __launch_bounds__(256) k_route_select(int T, int E, int k, int ksplit, int vocab, float routed_scale,
                                                      const float* __restrict__ part, const float* __restrict__ bias,
                                                      const int32_t* __restrict__ token_ids,
                                                      const int32_t* __restrict__ tid2eid, int32_t* __restrict__ topk_ids,
                                                      float* __restrict__ topk_w, uint32_t* status) {
  extern __shared__ float ssc[];  // [8 warps][E]
  pdl_wait();  // the partial logits come from the previous kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  float* s = ssc + size_t(warp) * E;
  // the splits are summed in split order; 32-expert slices in registers, four
  // splits' loads in flight at a time
  for (int e0 = 0; e0 < E; e0 += 256) {
    float z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) z[i] = 0.0f;
    for (int ks = 0; ks < ksplit; ks += 4) {
      float v[4][8];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = e0 + lane + 32 * i;
          v[j][i] = (ks + j < ksplit && e < E) ? __ldcg(part + (size_t(ks + j) * T + t) * E + e) : 0.0f;
        }
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] += v[j][i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = e0 + lane + 32 * i;
      if (e < E) s[e] = sqrt_softplus_f(z[i]);
    }
  }
  __syncwarp();
  if (HASH)
    select_hash_warp<true>(t, E, k, vocab, routed_scale, s, token_ids, tid2eid, topk_ids, topk_w, status);
  else
    select_learned<false>(t, E, k, routed_scale, s, bias, topk_ids, topk_w);
}

// bf16 [rows, cols] row-major, 128-byte swizzle, box {64, box_rows}.
bool rt_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {uint32_t(RK), box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int route_box_n(int E) { return std::min(RN, (E + 15) / 16 * 16); }

}  // namespace

int route_ksplit(const v4moe_config& c, int64_t T) {
  const int64_t tiles = (T + RT - 1) / RT * ((c.n_experts + RN - 1) / RN);
  const int nk = c.hidden / RK;
  int64_t ks = kRouteTargetCtas / std::max<int64_t>(tiles, 1);  // one wave
  ks = std::min<int64_t>(ks, std::max(1, std::min(16, nk / 2)));  // at least two stages per split
  return int(std::max<int64_t>(ks, 1));
}

cudaError_t launch_route(const v4moe_config& c, int T, const __nv_bfloat16* x, const __nv_bfloat16* gate,
                         const float* bias, const int32_t* token_ids, const int32_t* tid2eid, int32_t* topk_ids,
                         float* topk_w, float* part, uint32_t* status, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int E = c.n_experts, H = c.hidden;
  const int box_n = route_box_n(E);
  const int ks = route_ksplit(c, T);
  const int nk = H / RK, nk_per = (nk + ks - 1) / ks;
  CUtensorMap mX, mG;
  if (!rt_map(&mX, x, H, T, RT) || !rt_map(&mG, gate, H, E, box_n)) return cudaErrorInvalidValue;
  const int smem = kRStages * (kRA + box_n * RK * 2) + 256 + 1024;
  set_smem(k_route_gemm, smem);
  cudaError_t e = launch_kernel("route_gemm", k_route_gemm, dim3((T + RT - 1) / RT, ks, (E + box_n - 1) / box_n),
                                dim3(kRThreads), smem, st, false, T, E, nk, nk_per, box_n, part, status, mX, mG);
  if (e != cudaSuccess) return e;
  const size_t ssmem = size_t(8) * E * 4;
  if (token_ids) {
    set_smem(k_route_select<true>, ssmem);
    return launch_kernel("route_select_hash", k_route_select<true>, dim3((T + 7) / 8), dim3(256), ssmem, st, true, T,
                         E, c.top_k, ks, c.vocab, c.routed_scale, part, bias, token_ids, tid2eid, topk_ids, topk_w,
                         status);
  }
  set_smem(k_route_select<false>, ssmem);
  return launch_kernel("route_select", k_route_select<false>, dim3((T + 7) / 8), dim3(256), ssmem, st, true, T, E,
                       c.top_k, ks, c.vocab, c.routed_scale, part, bias, token_ids, tid2eid, topk_ids, topk_w, status);
}

}  // namespace v4moe
