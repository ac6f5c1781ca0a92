// Router of the DeepSeek-V4-Flash MoE layer ("Checked in its code" rows
// "Mixture of experts" and "Auxiliary-loss-free load balancing (selection
// bias)"; "config.json" scoring_func sqrtsoftplus, topk_method noaux_tc,
// norm_topk_prob, routed_scaling_factor; hash layers per "DeepSeek-V4-Flash
// export design", section "Source configuration").
//
// Learned routing, two kernels:
//  * k_route_scores: gate GEMV s[t, e] = sqrt(softplus(x[t] . gate[e])). One
//    CTA covers 32 experts x 8 tokens; each warp owns 4 experts and walks H in
//    16-byte pieces (8 bf16), with the 8 token rows staged in shared memory.
//    bf16 products are exact in fp32; accumulation is fp32.
//  * k_route_select: one warp per token; k rounds of a warp arg-max over
//    s + bias (value descending, expert id ascending on ties), ids emitted in
//    ascending order, weights = scale * s[id] / sum s[ids] from the unbiased
//    scores.
// Hash routing, one kernel (k_route_hash): one warp per token reads its
// tid2eid row and computes only the k needed gate dot products.
#include "launch.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kScoreTokens = 8;    // tokens per CTA
constexpr int kScoreExperts = 32;  // experts per CTA (4 per warp)
constexpr int kSelectWarps = 8;

__device__ __forceinline__ void fma_bf16x8(float& acc, const uint4& g, const uint4& x) {
  acc = fmaf(bf16_lo(g.x), bf16_lo(x.x), acc);
  acc = fmaf(bf16_hi(g.x), bf16_hi(x.x), acc);
  acc = fmaf(bf16_lo(g.y), bf16_lo(x.y), acc);
  acc = fmaf(bf16_hi(g.y), bf16_hi(x.y), acc);
  acc = fmaf(bf16_lo(g.z), bf16_lo(x.z), acc);
  acc = fmaf(bf16_hi(g.z), bf16_hi(x.z), acc);
  acc = fmaf(bf16_lo(g.w), bf16_lo(x.w), acc);
  acc = fmaf(bf16_hi(g.w), bf16_hi(x.w), acc);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(256) k_route_scores(int T, int H, int E,
                                                      const __nv_bfloat16* __restrict__ x,
                                                      const __nv_bfloat16* __restrict__ gate,
                                                      float* __restrict__ scores) {
  extern __shared__ __align__(16) uint4 xs[];  // [kScoreTokens][H/8]
  const int t0 = blockIdx.y * kScoreTokens;
  const int e0 = blockIdx.x * kScoreExperts;
  const int pieces = H / 8;
  for (int i = threadIdx.x; i < kScoreTokens * pieces; i += blockDim.x) {
    const int t = i / pieces, p = i % pieces;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t0 + t < T) v = reinterpret_cast<const uint4*>(x + size_t(t0 + t) * H)[p];
    xs[i] = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[4][kScoreTokens];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int t = 0; t < kScoreTokens; ++t) acc[a][t] = 0.0f;
  const uint4* grow[4];
  bool live[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int e = e0 + warp * 4 + a;
    live[a] = e < E;
    grow[a] = reinterpret_cast<const uint4*>(gate + size_t(live[a] ? e : 0) * H);
  }
  for (int p = lane; p < pieces; p += 32) {
    uint4 g[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) g[a] = __ldg(grow[a] + p);
#pragma unroll
    for (int t = 0; t < kScoreTokens; ++t) {
      const uint4 xv = xs[t * pieces + p];
#pragma unroll
      for (int a = 0; a < 4; ++a) fma_bf16x8(acc[a][t], g[a], xv);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int t = 0; t < kScoreTokens; ++t) acc[a][t] = warp_sum(acc[a][t]);
  if (lane == 0) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      if (!live[a]) continue;
      const int e = e0 + warp * 4 + a;
#pragma unroll
      for (int t = 0; t < kScoreTokens; ++t)
        if (t0 + t < T) scores[size_t(t0 + t) * E + e] = sqrt_softplus_f(acc[a][t]);
    }
  }
}

__global__ void __launch_bounds__(kSelectWarps * 32) k_route_select(
    int T, int E, int k, float routed_scale, const float* scores, const float* __restrict__ bias,
    int32_t* __restrict__ topk_ids, float* __restrict__ topk_w) {
  const int warp = threadIdx.x >> 5;
  const int t = blockIdx.x * kSelectWarps + warp;
  if (t >= T) return;
  select_learned_warp(t, E, k, routed_scale, scores + size_t(t) * E, bias, topk_ids, topk_w);
}

__global__ void __launch_bounds__(kSelectWarps * 32) k_route_hash(
    int T, int H, int E, int k, int vocab, float routed_scale, const __nv_bfloat16* __restrict__ x,
    const __nv_bfloat16* __restrict__ gate, const int32_t* __restrict__ token_ids,
    const int32_t* __restrict__ tid2eid, int32_t* __restrict__ topk_ids, float* __restrict__ topk_w,
    uint32_t* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelectWarps + warp;
  if (t >= T) return;
  const int tok = token_ids[t];
  const bool tok_ok = tok >= 0 && tok < vocab;
  int id[8];
  bool ok[8];
  bool any_bad = !tok_ok;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    id[r] = 0;
    ok[r] = false;
    if (r < k && tok_ok) {
      const int e = tid2eid[size_t(tok) * k + r];
      ok[r] = e >= 0 && e < E;
      id[r] = ok[r] ? e : 0;
      any_bad |= !ok[r];
    }
  }
  if (any_bad && lane == 0) atomicOr(status, tok_ok ? kStatusBadExpertId : kStatusBadTokenId);
  const uint4* xr = reinterpret_cast<const uint4*>(x + size_t(t) * H);
  float acc[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) acc[r] = 0.0f;
  for (int p = lane; p < H / 8; p += 32) {
    const uint4 xv = __ldg(xr + p);
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (r < k) fma_bf16x8(acc[r], __ldg(reinterpret_cast<const uint4*>(gate + size_t(id[r]) * H) + p), xv);
  }
  float sv[8];
  float sum = 0.0f;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    sv[r] = (r < k && ok[r]) ? sqrt_softplus_f(warp_sum(acc[r])) : 0.0f;
    sum += sv[r];
  }
  if (lane < k) {
    float myv = 0.0f;
    int myid = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (r == lane) {
        myv = sv[r];
        myid = id[r];
      }
    topk_ids[size_t(t) * k + lane] = myid;
    topk_w[size_t(t) * k + lane] = sum > 0.0f ? routed_scale * (myv / sum) : 0.0f;
  }
}

}  // namespace

cudaError_t launch_route(const v4moe_config& c, int T, const __nv_bfloat16* x,
                         const __nv_bfloat16* gate, const float* bias, const int32_t* token_ids,
                         const int32_t* tid2eid, int32_t* topk_ids, float* topk_w, float* scores,
                         uint32_t* status, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (token_ids) {
    const int blocks = (T + kSelectWarps - 1) / kSelectWarps;
    return launch_kernel("route_hash", k_route_hash, dim3(blocks), dim3(kSelectWarps * 32), 0, st, false,
                         T, c.hidden, c.n_experts, c.top_k, c.vocab, c.routed_scale, x, gate, token_ids,
                         tid2eid, topk_ids, topk_w, status);
  }
  const size_t smem = size_t(kScoreTokens) * c.hidden * 2;
  set_smem(k_route_scores, smem);
  dim3 grid((c.n_experts + kScoreExperts - 1) / kScoreExperts, (T + kScoreTokens - 1) / kScoreTokens);
  cudaError_t e = launch_kernel("route_scores", k_route_scores, grid, dim3(256), smem, st, false, T, c.hidden,
                                c.n_experts, x, gate, scores);
  if (e != cudaSuccess) return e;
  const int blocks = (T + kSelectWarps - 1) / kSelectWarps;
  return launch_kernel("route_select", k_route_select, dim3(blocks), dim3(kSelectWarps * 32), 0, st, false, T,
                       c.n_experts, c.top_k, c.routed_scale, (const float*)scores, bias, topk_ids, topk_w);
}

}  // namespace v4moe
