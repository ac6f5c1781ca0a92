// Fused routing for decode-sized batches: one launch computes the router
// scores, the top-k selection and weights, the token permutation and the
// activation layout the decode expert kernels read.
//
//  * every CTA (8 experts, one per warp) computes s[t, e] =
//    sqrt(softplus(x[t] . gate[e])) for all T tokens, with the token rows
//    staged 8 at a time in shared memory, and converts its share of the x rows
//    to the decode layout (f16, MMA K order, per-token power-of-two scale);
//  * the last CTA to finish (atomic ticket in the workspace, no waiting)
//    selects each token's experts and weights and sorts the slots by expert.
// The ticket is returned to zero by that last CTA, so the workspace is ready
// for the next call.
#include <cuda_fp16.h>

#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kPrepExperts = 8;   // experts per CTA, one per warp
constexpr int kPrepTokens = 8;    // token rows staged at once

struct PrepParams {
  int T, H, E, k, vocab;
  float routed_scale;
  const __nv_bfloat16* x;
  const __nv_bfloat16* gate;
  const float* bias;
  const int32_t* token_ids;
  const int32_t* tid2eid;
  int32_t* topk_ids;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_slot;
  int32_t* slot_pos;
  float* scores;
  __half* xlog;
  int* sigma;
  uint32_t* status;
  unsigned* ticket;
};

__device__ __forceinline__ void fma8(float& acc, const uint4& g, const uint4& x) {
  acc = fmaf(bf16_lo(g.x), bf16_lo(x.x), acc);
  acc = fmaf(bf16_hi(g.x), bf16_hi(x.x), acc);
  acc = fmaf(bf16_lo(g.y), bf16_lo(x.y), acc);
  acc = fmaf(bf16_hi(g.y), bf16_hi(x.y), acc);
  acc = fmaf(bf16_lo(g.z), bf16_lo(x.z), acc);
  acc = fmaf(bf16_hi(g.z), bf16_hi(x.z), acc);
  acc = fmaf(bf16_lo(g.w), bf16_lo(x.w), acc);
  acc = fmaf(bf16_hi(g.w), bf16_hi(x.w), acc);
}

__global__ void __launch_bounds__(256) k_dec_prep(PrepParams P) {
  extern __shared__ __align__(16) uint4 xs[];  // [kPrepTokens][H/8]
  __shared__ int cnt[1024];
  __shared__ int cursor[1024];
  __shared__ int is_last;
  // The expert kernels may launch now: their shared-expert CTAs stream
  // weights while the routing is computed.
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = P.H, T = P.T, E = P.E;
  const int pieces = H / 8;

  for (int t = blockIdx.x * 8 + warp; t < T; t += gridDim.x * 8)
    warp_row_to_decode_layout(P.x + size_t(t) * H, H, P.xlog + size_t(t) * H, P.sigma + t);

  const int e = blockIdx.x * kPrepExperts + warp;
  const uint4* grow = reinterpret_cast<const uint4*>(P.gate + size_t(e < E ? e : 0) * H);
  for (int t0 = 0; t0 < T; t0 += kPrepTokens) {
    __syncthreads();
    for (int i = threadIdx.x; i < kPrepTokens * pieces; i += blockDim.x) {
      const int tt = i / pieces, p = i % pieces;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t0 + tt < T) v = __ldg(reinterpret_cast<const uint4*>(P.x + size_t(t0 + tt) * H) + p);
      xs[i] = v;
    }
    __syncthreads();
    if (e < E) {
      float acc[kPrepTokens];
#pragma unroll
      for (int tt = 0; tt < kPrepTokens; ++tt) acc[tt] = 0.f;
#pragma unroll 4
      for (int p = lane; p < pieces; p += 32) {
        const uint4 g = __ldg(grow + p);
#pragma unroll
        for (int tt = 0; tt < kPrepTokens; ++tt) fma8(acc[tt], g, xs[tt * pieces + p]);
      }
#pragma unroll
      for (int tt = 0; tt < kPrepTokens; ++tt) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int tt = 0; tt < kPrepTokens; ++tt)
          if (t0 + tt < T) P.scores[size_t(t0 + tt) * E + e] = sqrt_softplus_f(acc[tt]);
      }
    }
  }

  // ---- last CTA: selection and permutation ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(P.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int t = warp; t < T; t += 8) {
    const float* s = P.scores + size_t(t) * E;
    if (P.token_ids)
      select_hash_warp(t, E, P.k, P.vocab, P.routed_scale, s, P.token_ids, P.tid2eid, P.topk_ids, P.topk_w,
                       P.status);
    else
      select_learned<true>(t, E, P.k, P.routed_scale, s, P.bias, P.topk_ids, P.topk_w);
  }
  __syncthreads();
  cta_permute(T * P.k, E, P.topk_ids, P.counts, P.offsets, P.sorted_slot, P.slot_pos, P.status, cnt, cursor);
  if (threadIdx.x == 0) *P.ticket = 0u;
}

}  // namespace

cudaError_t launch_dec_prep(const v4moe_config& c, int T, const __nv_bfloat16* x, const __nv_bfloat16* gate,
                            const float* bias, const int32_t* token_ids, const int32_t* tid2eid,
                            int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets,
                            int32_t* sorted_slot, int32_t* slot_pos, float* scores, __half* xlog, int* sigma,
                            uint32_t* status, unsigned* ticket, cudaStream_t st) {
  PrepParams P;
  P.T = T;
  P.H = c.hidden;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.vocab = c.vocab;
  P.routed_scale = c.routed_scale;
  P.x = x;
  P.gate = gate;
  P.bias = bias;
  P.token_ids = token_ids;
  P.tid2eid = tid2eid;
  P.topk_ids = topk_ids;
  P.topk_w = topk_w;
  P.counts = counts;
  P.offsets = offsets;
  P.sorted_slot = sorted_slot;
  P.slot_pos = slot_pos;
  P.scores = scores;
  P.xlog = xlog;
  P.sigma = sigma;
  P.status = status;
  P.ticket = ticket;
  const size_t smem = size_t(kPrepTokens) * c.hidden * 2;
  set_smem(k_dec_prep, smem);
  const int grid = (c.n_experts + kPrepExperts - 1) / kPrepExperts;
  return launch_kernel("dec_prep", k_dec_prep, dim3(grid), dim3(256), smem, st, false, P);
}

}  // namespace v4moe
