// Decode-sized expert path (at most 8 tokens, so at most 8 per expert):
// weight-streaming grouped GEMV on warp-level tensor-core MMA.
//
// What it computes ("Checked in its code" rows "SwiGLU feed-forward", "Shared
// expert"; "config.json" experts_w4a16 / linears_w8a16):
//   k_dec_w13: per group (routed expert or shared expert) and 8 output
//              channels j: [g; u] = W13[{j, I+j}] x_t for the group's tokens,
//              h_t[j] = silu(min(g, L)) * clamp(u, -L, L), stored as f16.
//   k_dec_w2:  per 16 output rows m (owner computes): the shared expert, then
//              every routed expert in ascending id: y = W2[m] h_t and
//              out[t, m] += w[t, j] * y (weight 1 for the shared expert); the
//              sum is written once as bf16. Fixed order, no output atomics in
//              global memory.
//
// How:
//  * Everything the CTA reads arrives by 1-D bulk async copies into shared
//    memory, tracked by mbarriers with bounded waits: the weight tile (16 rows,
//    one copy per row into a padded stride), its E8M0 scale rows, and the
//    activation rows, which the preparation step stored as f16 in the MMA's
//    K order (decode_logical_index) with a per-token power-of-two scale.
//  * Weights become exact f16 MMA operands: E2M1 pairs via
//    cvt.rn.f16x2.e2m1x2, int8 via an exact magic-number conversion. The E8M0
//    group scale is applied to the operand as an exact power of two relative
//    to the row's largest group exponent; the row factor multiplies the fp32
//    result. Exact for every group within 36 binades of its row's largest.
//  * mma.sync m16n8k16 with fp32 accumulation; the 8 warps split K and their
//    partial tiles are summed in warp order through shared memory.
//  * The shared expert's CTAs start streaming weights before the routing is
//    known (programmatic dependent launch); routed CTAs wait for it.
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kDW = 8;                 // warps per CTA
constexpr int kDThreads = kDW * 32;
constexpr int kTileRows = 16;          // weight rows per tile (one m16 MMA tile)
constexpr int kMaxStages = 4;
constexpr uint32_t kWaitTries = 1u << 20;

enum { kMx = 0, kS8 = 1 };

struct DecParams {
  int T, H, I, Is, E, k;
  float limit;
  int n_shared_ctas;             // k_dec_w13: CTAs [0, n) do the shared expert
  int stages;
  int stage_bytes;
  const __half* xlog;            // [T, H] decode layout
  const int* sigma;              // [T]
  const int32_t* offsets;
  const int32_t* sorted_slot;
  const float* topk_w;
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  const int8_t* sh13;
  const float* sh13_scale;
  const int8_t* sh2;
  const float* sh2_scale;
  __half* hlog;                  // [T*k, I] routed intermediates (sorted order, decode layout)
  __half* hslog;                 // [T, I_s] shared intermediates (decode layout)
  __nv_bfloat16* out;
  uint32_t* status;
};

__host__ __device__ inline int tile_stride(int fmt, int K) {
  const int rb = fmt == kMx ? K / 2 : K;
  return fmt == kMx ? rb + ((rb % 128 == 0) ? 64 : 0) : rb + 16;
}
__host__ __device__ inline int xs_stride(int K) { return K * 2 + 16; }
// Stage: weight tile followed by the 16 scale rows (MX only).
__host__ __device__ inline int stage_size(int fmt, int K) {
  return kTileRows * tile_stride(fmt, K) + (fmt == kMx ? kTileRows * (K / 32) : 0);
}

__device__ __forceinline__ size_t umin_(size_t a, size_t b) { return a < b ? a : b; }

__device__ __forceinline__ float pow2f(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((e + 127) << 23);
}

// Bounded wait that flags a timeout in the status word.
__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_wait_bounded(bar, parity, kWaitTries)) return true;
  atomicOr(status, kStatusTimeout);
  return false;
}

// Issue the copies of one weight tile (+ scale rows) into a stage; thread 0.
// rows[i] is the global row of tile row i; rows 0-7 and 8-15 are each
// contiguous, so their scale rows come in two copies.
__device__ __forceinline__ void issue_tile(char* stage, int fmt, int K, const uint8_t* base,
                                           const uint8_t* scales, const int* rows, uint64_t* bar) {
  const int rb = fmt == kMx ? K / 2 : K;
  const int ws = tile_stride(fmt, K);
  const int G = K / 32;
  const uint32_t bytes = uint32_t(kTileRows * rb + (fmt == kMx ? kTileRows * G : 0));
  mbar_arrive_expect_tx(bar, bytes);
#pragma unroll 1
  for (int i = 0; i < kTileRows; ++i) bulk_g2s(stage + i * ws, base + size_t(rows[i]) * rb, uint32_t(rb), bar);
  if (fmt == kMx) {
    char* sc = stage + kTileRows * ws;
    bulk_g2s(sc, scales + size_t(rows[0]) * G, uint32_t(8 * G), bar);
    bulk_g2s(sc + 8 * G, scales + size_t(rows[8]) * G, uint32_t(8 * G), bar);
  }
}

// Largest E8M0 exponent of each of the 16 scale rows in shared memory.
__device__ __forceinline__ void row_max_exp(const uint8_t* sc, int G, int* rowx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < kTileRows; r += kDW) {
    int m = 0;
    for (int g = lane; g < G; g += 32) m = max(m, int(sc[r * G + g]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) rowx[r] = m;
  }
}

// One warp's share (K blocks warp, warp + 8, ...) of a 16-row tile times the
// staged activation rows (one n8 tile). acc: fp32 C fragment (rows g, g+8;
// token columns 2t, 2t+1).
template <int FMT>
__device__ __forceinline__ void warp_tile_mma(const char* wt, int wstride, const uint8_t* sc, const char* xs,
                                              int K, int nrows, const int* rowx, float acc[4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = K / 32;
  const int nblk = K / 128;
  int tok = min(lane & 7, nrows - 1);
  const uint32_t xaddr = smem_u32(xs + size_t(tok) * xs_stride(K)) + ((lane >> 3) & 1) * 16 + (lane >> 4) * 32;
  const int xa = FMT == kMx ? rowx[g] : 0;
  const int xb = FMT == kMx ? rowx[g + 8] : 0;
  for (int b = warp; b < nblk; b += kDW) {
    uint32_t A[8][4];
    if (FMT == kMx) {
      const uint4 qa = *reinterpret_cast<const uint4*>(wt + g * wstride + b * 64 + 16 * t);
      const uint4 qb = *reinterpret_cast<const uint4*>(wt + (g + 8) * wstride + b * 64 + 16 * t);
      const uint32_t sa = f16_pow2_bits(int(sc[g * G + 4 * b + t]) - xa + 13) * 0x10001u;
      const uint32_t sb = f16_pow2_bits(int(sc[(g + 8) * G + 4 * b + t]) - xb + 13) * 0x10001u;
      const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
      const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        uint32_t fa[4], fb[4];
        e2m1x8_to_f16x2(wa[wi], fa);
        e2m1x8_to_f16x2(wb[wi], fb);
        A[2 * wi][0] = hmul2_u32(fa[0], sa);
        A[2 * wi][1] = hmul2_u32(fb[0], sb);
        A[2 * wi][2] = hmul2_u32(fa[1], sa);
        A[2 * wi][3] = hmul2_u32(fb[1], sb);
        A[2 * wi + 1][0] = hmul2_u32(fa[2], sa);
        A[2 * wi + 1][1] = hmul2_u32(fb[2], sb);
        A[2 * wi + 1][2] = hmul2_u32(fa[3], sa);
        A[2 * wi + 1][3] = hmul2_u32(fb[3], sb);
      }
    } else {
      const uint4* pa = reinterpret_cast<const uint4*>(wt + g * wstride + b * 128 + 32 * t);
      const uint4* pb = reinterpret_cast<const uint4*>(wt + (g + 8) * wstride + b * 128 + 32 * t);
      const uint4 qa0 = pa[0], qa1 = pa[1], qb0 = pb[0], qb1 = pb[1];
      const uint32_t wa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
      const uint32_t wb[8] = {qb0.x, qb0.y, qb0.z, qb0.w, qb1.x, qb1.y, qb1.z, qb1.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        s8x4_to_f16x2(wa[s], A[s][0], A[s][2]);
        s8x4_to_f16x2(wb[s], A[s][1], A[s][3]);
      }
    }
#pragma unroll
    for (int sp = 0; sp < 4; ++sp) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(b0, b1, b2, b3, xaddr + (b * 128 + sp * 32) * 2);
      mma_16816_f16(acc, A[2 * sp], b0, b1);
      mma_16816_f16(acc, A[2 * sp + 1], b2, b3);
    }
  }
}

// Sum the 8 warps' C fragments in warp order; result valid in warp 0.
__device__ __forceinline__ void reduce_warps(float acc[4], float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i) red[(warp * 4 + i) * 32 + lane] = acc[i];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float s = 0.f;
      for (int w = 0; w < kDW; ++w) s += red[(w * 4 + i) * 32 + lane];
      acc[i] = s;
    }
  }
}

// Compact list of non-empty routed experts in ascending id (one warp).
__device__ __forceinline__ int build_hit_list(const int32_t* offsets, int E, int* list) {
  const int lane = threadIdx.x & 31;
  int n = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const bool hit = e < E && offsets[e + 1] > offsets[e];
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (hit) list[n + __popc(m & ((1u << lane) - 1u))] = e;
    n += __popc(m);
  }
  return n;
}

struct SmemDec {
  uint64_t bars[kMaxStages];
  uint64_t xbar;
  int rowx[kMaxStages][kTileRows];
  int rows[kMaxStages][kTileRows];
  int nlist;
};

// ------------------------------------------------------------------ w13

__global__ void __launch_bounds__(kDThreads) k_dec_w13(DecParams P) {
  extern __shared__ __align__(128) char smem[];
  SmemDec& S = *reinterpret_cast<SmemDec*>(smem);
  int* list = reinterpret_cast<int*>(smem + 1024);
  float* red = reinterpret_cast<float*>(smem + 1024 + ((P.E + 1) * 4 + 127) / 128 * 128);
  char* stages = reinterpret_cast<char*>(red + kDW * 4 * 32);
  char* xs = stages + size_t(P.stages) * P.stage_bytes;
  const int H = P.H, T = P.T;
  const bool shared_cta = int(blockIdx.x) < P.n_shared_ctas;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int fmt = shared_cta ? kS8 : kMx;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) mbar_init(&S.bars[s], 1);
    mbar_init(&S.xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ---- work range ----
  int n_routed = 0, it0 = 0, it1 = 0, blk = 0;
  if (shared_cta) {
    blk = P.Is / 8;
    const int per = (blk + P.n_shared_ctas - 1) / P.n_shared_ctas;
    it0 = blockIdx.x * per;
    it1 = min(blk, it0 + per);
  } else {
    pdl_wait();  // routing comes from the preparation kernel
    if (warp == 0) {
      const int n = build_hit_list(P.offsets, P.E, list);
      if (lane == 0) S.nlist = n;
    }
    __syncthreads();
    n_routed = S.nlist;
    blk = P.I / 8;
    const int n_items = n_routed * blk;
    const int ctas = gridDim.x - P.n_shared_ctas;
    const int per = (n_items + ctas - 1) / ctas;
    it0 = (blockIdx.x - P.n_shared_ctas) * per;
    it1 = min(n_items, it0 + per);
  }
  const int Ig = shared_cta ? P.Is : P.I;
  auto item_group = [&](int it) { return shared_cta ? P.E : list[it / blk]; };
  auto issue = [&](int it, int s) {  // thread 0
    const int grp = item_group(it);
    const int j0 = (it % blk) * 8;
    for (int i = 0; i < kTileRows; ++i) S.rows[s][i] = i < 8 ? j0 + i : Ig + j0 + (i - 8);
    const uint8_t* base = shared_cta ? reinterpret_cast<const uint8_t*>(P.sh13)
                                     : P.w13_codes + size_t(grp) * 2 * P.I * (H / 2);
    const uint8_t* scl = shared_cta ? nullptr : P.w13_scales + size_t(grp) * 2 * P.I * (H / 32);
    issue_tile(stages + size_t(s) * P.stage_bytes, fmt, H, base, scl, S.rows[s], &S.bars[s]);
  };
  if (it0 < it1 && threadIdx.x == 0)
    for (int s = 0; s < P.stages && it0 + s < it1; ++s) issue(it0 + s, s);
  // Ask for every later tile of this CTA now, into L2: the whole weight stream
  // of the kernel is then in flight at once and the ring's copies hit L2.
  if (warp == 1) {
    for (int it = it0 + P.stages + lane; it < it1; it += 32) {
      const int grp = item_group(it);
      const int j0 = (it % blk) * 8;
      if (shared_cta) {
        const uint8_t* b = reinterpret_cast<const uint8_t*>(P.sh13);
        prefetch_l2_bulk(b + size_t(j0) * H, uint32_t(8 * H));
        prefetch_l2_bulk(b + size_t(Ig + j0) * H, uint32_t(8 * H));
      } else {
        const uint8_t* b = P.w13_codes + size_t(grp) * 2 * P.I * (H / 2);
        const uint8_t* sc = P.w13_scales + size_t(grp) * 2 * P.I * (H / 32);
        prefetch_l2_bulk(b + size_t(j0) * (H / 2), uint32_t(8 * (H / 2)));
        prefetch_l2_bulk(b + size_t(Ig + j0) * (H / 2), uint32_t(8 * (H / 2)));
        prefetch_l2_bulk(sc + size_t(j0) * (H / 32), uint32_t(8 * (H / 32)));
        prefetch_l2_bulk(sc + size_t(Ig + j0) * (H / 32), uint32_t(8 * (H / 32)));
      }
    }
  }
  // The down projection of the same experts streams next: start moving its
  // weights into L2 while this kernel runs (the routed CTAs split the hit
  // experts' W2 blocks; the shared CTAs split the shared expert's).
  if (warp == 2 && lane == 0) {
    const int nctas = shared_cta ? P.n_shared_ctas : int(gridDim.x) - P.n_shared_ctas;
    const int me = shared_cta ? int(blockIdx.x) : int(blockIdx.x) - P.n_shared_ctas;
    if (shared_cta) {
      const size_t total = size_t(H) * P.Is;
      const size_t per = (total / nctas + 15) / 16 * 16;
      const size_t a = size_t(me) * per;
      if (a < total) prefetch_l2_range(reinterpret_cast<const uint8_t*>(P.sh2) + a, umin_(per, total - a));
    } else if (n_routed > 0) {
      const size_t codes = size_t(H) * (P.I / 2), scl = size_t(H) * (P.I / 32);
      const size_t per_e = codes + scl;
      const size_t total = per_e * n_routed;
      const size_t per = (total / nctas + 15) / 16 * 16;
      size_t a = size_t(me) * per;
      const size_t b = umin_(total, a + per);
      while (a < b) {
        const int li = int(a / per_e);
        size_t off = a - size_t(li) * per_e;
        const size_t n = umin_(b - a, per_e - off);
        const int e = list[li];
        if (off < codes) {
          const size_t nc = umin_(n, codes - off);
          prefetch_l2_range(P.w2_codes + size_t(e) * codes + off, nc);
          if (n > nc) prefetch_l2_range(P.w2_scales + size_t(e) * scl, n - nc);
        } else {
          prefetch_l2_range(P.w2_scales + size_t(e) * scl + (off - codes), n);
        }
        a += n;
      }
    }
  }
  if (shared_cta) pdl_wait();  // the activations come from the preparation kernel
  if (it0 >= it1) return;

  int staged = -1;
  uint32_t xphase = 0;
  for (int it = it0; it < it1; ++it) {
    const int i = it - it0;
    const int s = i % P.stages;
    const uint32_t parity = uint32_t(i / P.stages) & 1u;
    const int grp = item_group(it);
    const int j0 = (it % blk) * 8;
    const int r0 = shared_cta ? 0 : P.offsets[grp];
    const int n = shared_cta ? T : P.offsets[grp + 1] - r0;
    if (grp != staged) {
      __syncthreads();  // readers of the previous activations are done
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&S.xbar, uint32_t(n * H * 2));
        for (int r = 0; r < n; ++r) {
          const int tok = shared_cta ? r : P.sorted_slot[r0 + r] / P.k;
          bulk_g2s(xs + size_t(r) * xs_stride(H), P.xlog + size_t(tok) * H, uint32_t(H * 2), &S.xbar);
        }
      }
      if (!wait_or_flag(&S.xbar, xphase, P.status)) break;
      xphase ^= 1u;
      staged = grp;
    }
    if (!wait_or_flag(&S.bars[s], parity, P.status)) break;
    const char* st = stages + size_t(s) * P.stage_bytes;
    const uint8_t* sc = reinterpret_cast<const uint8_t*>(st + kTileRows * tile_stride(fmt, H));
    if (fmt == kMx) row_max_exp(sc, H / 32, S.rowx[s]);
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (fmt == kMx)
      warp_tile_mma<kMx>(st, tile_stride(kMx, H), sc, xs, H, n, S.rowx[s], acc);
    else
      warp_tile_mma<kS8>(st, tile_stride(kS8, H), nullptr, xs, H, n, S.rowx[s], acc);
    reduce_warps(acc, red);
    if (warp == 0) {
      float fg, fu;
      if (fmt == kMx) {
        fg = pow2f(S.rowx[s][g] - 127 - 13);
        fu = pow2f(S.rowx[s][g + 8] - 127 - 13);
      } else {
        fg = __ldg(P.sh13_scale + j0 + g);
        fu = __ldg(P.sh13_scale + Ig + j0 + g);
      }
      __half* hout = shared_cta ? P.hslog : P.hlog;
      const int L = decode_logical_index(j0 + g);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int nn = 2 * t + q;
        if (nn < n) {
          const int tok = shared_cta ? nn : P.sorted_slot[r0 + nn] / P.k;
          const float inv = pow2f(-P.sigma[tok]);
          const float gv = acc[q] * fg * inv;
          const float uv = acc[2 + q] * fu * inv;
          hout[size_t(r0 + nn) * Ig + L] = __float2half_rn(clamped_swiglu_f(gv, uv, P.limit));
        }
      }
    }
    __syncthreads();  // every warp is done with stage s
    if (threadIdx.x == 0 && it + P.stages < it1) issue(it + P.stages, s);
  }
  // Only reached early after a timeout: give the copies still in flight into
  // this CTA's shared memory a bounded wait before leaving.
  if (threadIdx.x == 0)
    for (int s = 0; s < P.stages; ++s) mbar_wait_bounded(&S.bars[s], 0, 1);
}

// ------------------------------------------------------------------ w2 + combine

__global__ void __launch_bounds__(kDThreads) k_dec_w2(DecParams P) {
  extern __shared__ __align__(128) char smem[];
  SmemDec& S = *reinterpret_cast<SmemDec*>(smem);
  int* list = reinterpret_cast<int*>(smem + 1024);
  float* red = reinterpret_cast<float*>(smem + 1024 + ((P.E + 2) * 4 + 127) / 128 * 128);
  float* oacc = red + kDW * 4 * 32;                                   // [T][16]
  char* stages = reinterpret_cast<char*>(oacc) + ((P.T * kTileRows * 4 + 127) / 128) * 128;
  char* xs = stages + size_t(P.stages) * P.stage_bytes;
  const int H = P.H, T = P.T;
  const int m0 = blockIdx.x * kTileRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  for (int i = threadIdx.x; i < T * kTileRows; i += kDThreads) oacc[i] = 0.f;
  if (threadIdx.x < kTileRows)
    for (int s = 0; s < kMaxStages; ++s) S.rows[s][threadIdx.x] = m0 + threadIdx.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) mbar_init(&S.bars[s], 1);
    mbar_init(&S.xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool has_shared = P.Is > 0;
  auto issue = [&](int gi, int s) {  // thread 0
    const bool sh = gi == P.E;
    const int Kg = sh ? P.Is : P.I;
    const uint8_t* base = sh ? reinterpret_cast<const uint8_t*>(P.sh2) : P.w2_codes + size_t(gi) * H * (P.I / 2);
    const uint8_t* scl = sh ? nullptr : P.w2_scales + size_t(gi) * H * (P.I / 32);
    issue_tile(stages + size_t(s) * P.stage_bytes, sh ? kS8 : kMx, Kg, base, scl, S.rows[s], &S.bars[s]);
  };
  // The shared expert goes first; its weights do not depend on the routing.
  if (threadIdx.x == 0 && has_shared) issue(P.E, 0);
  pdl_wait();  // h and the routing come from the previous kernels
  if (warp == 0) {
    if (has_shared && lane == 0) list[0] = P.E;
    const int n = build_hit_list(P.offsets, P.E, list + (has_shared ? 1 : 0));
    if (lane == 0) S.nlist = n + (has_shared ? 1 : 0);
  }
  __syncthreads();
  const int nl = S.nlist;
  if (threadIdx.x == 0)
    for (int s = has_shared ? 1 : 0; s < P.stages && s < nl; ++s) issue(list[s], s);

  uint32_t xphase = 0;
  bool ok = true;
  for (int li = 0; li < nl && ok; ++li) {
    const int s = li % P.stages;
    const uint32_t parity = uint32_t(li / P.stages) & 1u;
    const int gi = list[li];
    const bool sh = gi == P.E;
    const int fmt = sh ? kS8 : kMx;
    const int Kg = sh ? P.Is : P.I;
    const int r0 = sh ? 0 : P.offsets[gi];
    const int n = sh ? T : P.offsets[gi + 1] - r0;
    if (threadIdx.x == 0) {
      const __half* src = sh ? P.hslog : P.hlog;
      mbar_arrive_expect_tx(&S.xbar, uint32_t(n * Kg * 2));
      for (int r = 0; r < n; ++r)
        bulk_g2s(xs + size_t(r) * xs_stride(Kg), src + size_t(r0 + r) * Kg, uint32_t(Kg * 2), &S.xbar);
    }
    ok = wait_or_flag(&S.bars[s], parity, P.status);
    ok = wait_or_flag(&S.xbar, xphase, P.status) && ok;
    xphase ^= 1u;
    if (!ok) break;
    const char* st = stages + size_t(s) * P.stage_bytes;
    const uint8_t* sc = reinterpret_cast<const uint8_t*>(st + kTileRows * tile_stride(fmt, Kg));
    if (fmt == kMx) row_max_exp(sc, Kg / 32, S.rowx[s]);
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (fmt == kMx)
      warp_tile_mma<kMx>(st, tile_stride(kMx, Kg), sc, xs, Kg, n, S.rowx[s], acc);
    else
      warp_tile_mma<kS8>(st, tile_stride(kS8, Kg), nullptr, xs, Kg, n, S.rowx[s], acc);
    reduce_warps(acc, red);
    if (warp == 0) {
      float fa, fb;
      if (fmt == kMx) {
        fa = pow2f(S.rowx[s][g] - 127 - 13);
        fb = pow2f(S.rowx[s][g + 8] - 127 - 13);
      } else {
        fa = __ldg(P.sh2_scale + m0 + g);
        fb = __ldg(P.sh2_scale + m0 + g + 8);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int nn = 2 * t + q;
        if (nn < n) {
          int tok;
          float wgt;
          if (sh) {
            tok = nn;
            wgt = 1.0f;
          } else {
            const int slot = P.sorted_slot[r0 + nn];
            tok = slot / P.k;
            wgt = P.topk_w[slot];
          }
          atomicAdd(&oacc[tok * kTileRows + g], wgt * (acc[q] * fa));
          atomicAdd(&oacc[tok * kTileRows + g + 8], wgt * (acc[2 + q] * fb));
        }
      }
    }
    __syncthreads();  // every warp is done with stage s and the activations
    if (threadIdx.x == 0 && li + P.stages < nl) issue(list[li + P.stages], s);
  }
  if (!ok) {
    if (threadIdx.x == 0)
      for (int s = 0; s < P.stages; ++s) mbar_wait_bounded(&S.bars[s], 0, 1);
    return;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < T * kTileRows; i += kDThreads) {
    const int tok = i / kTileRows, r = i % kTileRows;
    P.out[size_t(tok) * H + m0 + r] = __float2bfloat16_rn(oacc[i]);
  }
}

// x -> decode layout for the forward path that does not go through the fused
// preparation kernel (routing supplied by the caller).
__global__ void __launch_bounds__(256) k_dec_xlog(int T, int H, const __nv_bfloat16* __restrict__ x,
                                                  __half* __restrict__ xlog, int* __restrict__ sigma) {
  const int warp = threadIdx.x >> 5;
  const int tt = blockIdx.x * 8 + warp;
  if (tt < T) warp_row_to_decode_layout(x + size_t(tt) * H, H, xlog + size_t(tt) * H, sigma + tt);
}

size_t w13_fixed(const v4moe_config& c) {
  return 1024 + size_t((c.n_experts + 1) * 4 + 127) / 128 * 128 + size_t(kDW) * 4 * 32 * 4;
}
size_t w2_fixed(const v4moe_config& c, int T) {
  return 1024 + size_t((c.n_experts + 2) * 4 + 127) / 128 * 128 + size_t(kDW) * 4 * 32 * 4 +
         size_t((T * kTileRows * 4 + 127) / 128) * 128;
}
int w13_stage(const v4moe_config& c) {
  return std::max(stage_size(kMx, c.hidden), c.shared_inter > 0 ? stage_size(kS8, c.hidden) : 0);
}
int w2_stage(const v4moe_config& c) {
  return std::max(stage_size(kMx, c.inter), c.shared_inter > 0 ? stage_size(kS8, c.shared_inter) : 0);
}
constexpr size_t kSmemMax = 227 * 1024;

// Stages that fit next to the fixed part and the activation rows (up to
// kMaxStages); `prefer_bytes` caps the size when that still leaves
// `min_stages` stages (so that two CTAs share an SM).
void plan(size_t fixed, size_t stage, size_t acts, size_t prefer_bytes, int min_stages, int* stages,
          size_t* bytes) {
  const size_t room = kSmemMax > fixed + acts ? kSmemMax - fixed - acts : 0;
  int s = int(std::min<size_t>(kMaxStages, room / stage));
  const size_t pref_room = prefer_bytes > fixed + acts ? prefer_bytes - fixed - acts : 0;
  const int s_pref = int(std::min<size_t>(kMaxStages, pref_room / stage));
  if (s_pref >= min_stages) s = std::min(s, s_pref);
  *stages = s;
  *bytes = fixed + acts + size_t(s) * stage;
}

}  // namespace

bool dec_supported(const v4moe_config& c, int T) {
  if (T > kDecodeMaxTokens || T < 1) return false;
  int s13, s2;
  size_t b13, b2;
  plan(w13_fixed(c), w13_stage(c), size_t(T) * xs_stride(c.hidden), kSmemMax, 2, &s13, &b13);
  plan(w2_fixed(c, T), w2_stage(c), size_t(T) * xs_stride(std::max(c.inter, c.shared_inter)), kSmemMax, 2,
       &s2, &b2);
  return s13 >= 2 && s2 >= 2;
}

cudaError_t launch_dec_xlog(const v4moe_config& c, int T, const __nv_bfloat16* x, __half* xlog, int* sigma,
                            cudaStream_t st) {
  return launch_kernel("dec_xlog", k_dec_xlog, dim3((T + 7) / 8), dim3(256), 0, st, false, T, c.hidden, x, xlog,
                       sigma);
}

cudaError_t launch_forward_dec(const ForwardArgs& a, const __half* xlog, const int* sigma, cudaStream_t st) {
  const v4moe_config& c = a.c;
  if (a.T == 0) return cudaSuccess;
  DecParams P;
  P.T = a.T;
  P.H = c.hidden;
  P.I = c.inter;
  P.Is = c.shared_inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.limit = c.swiglu_limit;
  P.xlog = xlog;
  P.sigma = sigma;
  P.offsets = a.offsets;
  P.sorted_slot = a.sorted_slot;
  P.topk_w = a.topk_w;
  P.w13_codes = a.w.w13_codes;
  P.w13_scales = a.w.w13_scales;
  P.w2_codes = a.w.w2_codes;
  P.w2_scales = a.w.w2_scales;
  P.sh13 = a.w.sh_w13;
  P.sh13_scale = a.w.sh_w13_scale;
  P.sh2 = a.w.sh_w2;
  P.sh2_scale = a.w.sh_w2_scale;
  P.hlog = reinterpret_cast<__half*>(a.h);
  P.hslog = reinterpret_cast<__half*>(a.hs);
  P.out = a.out;
  P.status = a.status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

  // ---- w13: one persistent CTA per SM; a share of them on the shared expert,
  // sized by its fraction of the weight bytes (routed experts hit <= T*k).
  int stages13;
  size_t smem13;
  plan(w13_fixed(c), w13_stage(c), size_t(a.T) * xs_stride(c.hidden), kSmemMax, 2, &stages13, &smem13);
  const int grid13 = sms;
  int nsh = 0;
  if (c.shared_inter > 0) {
    const double sh_bytes = double(2 * c.shared_inter) * c.hidden;
    const double rt_bytes = double(std::min(c.n_experts, a.T * c.top_k)) * (2.0 * c.inter * c.hidden / 2);
    nsh = int(std::lround(grid13 * sh_bytes / (sh_bytes + rt_bytes)));
    nsh = std::max(1, std::min(grid13 - 1, nsh));
  }
  P.n_shared_ctas = nsh;
  P.stages = stages13;
  P.stage_bytes = w13_stage(c);
  set_smem(k_dec_w13, smem13);
  cudaError_t e = launch_kernel("dec_w13", k_dec_w13, dim3(grid13), dim3(kDThreads), smem13, st, true, P);
  if (e != cudaSuccess) return e;

  // ---- w2 + combine: one CTA per 16 output rows; aim for two CTAs per SM.
  int stages2;
  size_t smem2;
  plan(w2_fixed(c, a.T), w2_stage(c), size_t(a.T) * xs_stride(std::max(c.inter, c.shared_inter)),
       kSmemMax / 2 - 1024, 3, &stages2, &smem2);
  P.stages = stages2;
  P.stage_bytes = w2_stage(c);
  set_smem(k_dec_w2, smem2);
  return launch_kernel("dec_w2", k_dec_w2, dim3(c.hidden / kTileRows), dim3(kDThreads), smem2, st, true, P);
}

}  // namespace v4moe
