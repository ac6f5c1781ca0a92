// Router of the DeepSeek-V4-Flash MoE layer ("Checked in its code" rows
// "Mixture of experts" and "Auxiliary-loss-free load balancing (selection
// bias)"; "config.json" scoring_func sqrtsoftplus, topk_method noaux_tc,
// norm_topk_prob, routed_scaling_factor; hash layers per "DeepSeek-V4-Flash
// export design", section "Source configuration").
//
//  * k_route_mma: per CTA 32 tokens x all experts; the gate
//    GEMV runs as a bf16 tensor-core GEMM (exact products, fp32 sums), and
//    sqrt(softplus), the biased top-k (ties to the lower id, ids ascending)
//    and the weights (unbiased scores, normalised, x routed_scaling_factor)
//    follow from shared memory in the same kernel.
//    Hash routing (first layers) uses the same kernel: the scores at the
//    tid2eid row's experts give the weights.
// The decode-sized fused variant is in decode_prep.cu.
#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {


// Learned routing on tensor cores: per CTA 32 tokens x all experts,
// logits = x . gate^T with bf16 mma.sync (exact products, fp32 sums), then
// sqrt(softplus) and the biased top-k selection from shared memory.
// K is walked in 64-element slices, double-buffered with cp.async; rows are
// stored with their 16-byte chunks XOR-swizzled by (row & 7) so that the
// ldmatrix reads are conflict-free.
constexpr int kRmTok = 32;     // tokens per CTA
constexpr int kRmExp = 256;    // experts per pass (8 warps x 32)
constexpr int kRmBK = 64;

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4)); }

template <bool HASH>
__global__ void __launch_bounds__(256) k_route_mma(int T, int H, int E, int k, int vocab, float routed_scale,
                                                   const __nv_bfloat16* __restrict__ x,
                                                   const __nv_bfloat16* __restrict__ gate,
                                                   const float* __restrict__ bias,
                                                   const int32_t* __restrict__ token_ids,
                                                   const int32_t* __restrict__ tid2eid,
                                                   int32_t* __restrict__ topk_ids, float* __restrict__ topk_w,
                                                   uint32_t* status) {
  extern __shared__ __align__(128) char sm[];
  char* As = sm;                                   // [2][32 rows][128 B]
  char* Bs = sm + 2 * kRmTok * 128;                // [2][256 rows][128 B]
  float* sc = reinterpret_cast<float*>(Bs + 2 * kRmExp * 128);  // [32][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRmTok;
  const int nk = H / kRmBK;
  for (int e0 = 0; e0 < E; e0 += kRmExp) {
    auto load = [&](int kb, int buf) {
      char* a = As + buf * kRmTok * 128;
      char* b = Bs + buf * kRmExp * 128;
      {  // x: 32 rows x 8 chunks, one per thread
        const int row = threadIdx.x >> 3, ch = threadIdx.x & 7;
        const bool ok = t0 + row < T;
        cp_async16_zfill(a + swz(row, ch), x + size_t(ok ? t0 + row : 0) * H + kb * kRmBK + ch * 8, ok);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // gate: 256 rows x 8 chunks
        const int idx = threadIdx.x + i * 256;
        const int row = idx >> 3, ch = idx & 7;
        const bool ok = e0 + row < E;
        cp_async16_zfill(b + swz(row, ch), gate + size_t(ok ? e0 + row : 0) * H + kb * kRmBK + ch * 8, ok);
      }
      cp_async_commit();
    };
    float acc[2][4][4] = {};
    load(0, 0);
    for (int kb = 0; kb < nk; ++kb) {
      if (kb + 1 < nk) {
        load(kb + 1, (kb + 1) & 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint32_t a = smem_u32(As + (kb & 1) * kRmTok * 128);
      const uint32_t b = smem_u32(Bs + (kb & 1) * kRmExp * 128);
#pragma unroll
      for (int kk = 0; kk < kRmBK / 16; ++kk) {
        uint32_t af[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          ldmatrix_x4(af[mt][0], af[mt][1], af[mt][2], af[mt][3], a + swz(row, kk * 2 + (lane >> 4)));
        }
#pragma unroll
        for (int np = 0; np < 2; ++np) {  // pairs of n8 tiles
          const int row = warp * 32 + np * 16 + (lane & 7) + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(b0, b1, b2, b3, b + swz(row, kk * 2 + ((lane >> 3) & 1)));
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_16816_bf16(acc[mt][2 * np], af[mt], b0, b1);
            mma_16816_bf16(acc[mt][2 * np + 1], af[mt], b2, b3);
          }
        }
      }
      __syncthreads();
    }
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tok = mt * 16 + g + (i >> 1) * 8;
          const int e = e0 + warp * 32 + nt * 8 + 2 * t + (i & 1);
          if (e < E) sc[tok * E + e] = sqrt_softplus_f(acc[mt][nt][i]);
        }
  }
  __syncthreads();
  for (int tt = warp; tt < kRmTok; tt += 8) {
    if (t0 + tt >= T) continue;
    if (HASH)
      select_hash_warp<true>(t0 + tt, E, k, vocab, routed_scale, sc + tt * E, token_ids, tid2eid, topk_ids, topk_w,
                             status);
    else
      select_learned<false>(t0 + tt, E, k, routed_scale, sc + tt * E, bias, topk_ids, topk_w);
  }
}

}  // namespace

cudaError_t launch_route(const v4moe_config& c, int T, const __nv_bfloat16* x,
                         const __nv_bfloat16* gate, const float* bias, const int32_t* token_ids,
                         const int32_t* tid2eid, int32_t* topk_ids, float* topk_w, float* scores,
                         uint32_t* status, cudaStream_t st) {
  (void)scores;
  if (T == 0) return cudaSuccess;
  const size_t smem = size_t(2) * (kRmTok + kRmExp) * 128 + size_t(kRmTok) * c.n_experts * 4;
  const dim3 grid((T + kRmTok - 1) / kRmTok);
  if (token_ids) {
    set_smem(k_route_mma<true>, smem);
    return launch_kernel("route_mma_hash", k_route_mma<true>, grid, dim3(256), smem, st, false, T, c.hidden,
                         c.n_experts, c.top_k, c.vocab, c.routed_scale, x, gate, bias, token_ids, tid2eid, topk_ids,
                         topk_w, status);
  }
  set_smem(k_route_mma<false>, smem);
  return launch_kernel("route_mma", k_route_mma<false>, grid, dim3(256), smem, st, false, T, c.hidden, c.n_experts,
                       c.top_k, c.vocab, c.routed_scale, x, gate, bias, token_ids, tid2eid, topk_ids, topk_w, status);
}

}  // namespace v4moe
