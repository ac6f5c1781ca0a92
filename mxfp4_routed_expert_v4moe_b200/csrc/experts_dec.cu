// Decode-sized expert path (few tokens per expert): weight-streaming grouped
// GEMV/GEMM on warp-level tensor-core MMA.
//
// What it computes ("Checked in its code" rows "SwiGLU feed-forward", "Shared
// expert"; "config.json" experts_w4a16 / linears_w8a16):
//   k_dec_w13: per group (routed expert or shared expert) and 8 output
//              channels j: [g; u] = W13[{j, I+j}] x_t for the group's tokens,
//              h_t[j] = silu(min(g, L)) * clamp(u, -L, L), stored as f16.
//   k_dec_w2:  per 16 output rows m (owner computes): for every group in
//              ascending expert id, then the shared expert, y = W2[m] h_t and
//              out[t, m] += w[t, j] * y (weight 1 for the shared expert);
//              the sum is written once as bf16. No atomics, fixed order.
//
// How:
//  * The CTA's weight tile (16 rows x K) is brought into shared memory with
//    one 1-D bulk async copy per row (padded row stride for conflict-free
//    reads), completion tracked by an mbarrier with a bounded wait.
//  * Weights become exact f16 MMA operands: E2M1 pairs via
//    cvt.rn.f16x2.e2m1x2, int8 via an exact magic-number conversion. The
//    E8M0 group scale is applied to the operand as an exact power of two
//    relative to the row's largest group exponent; the row factor is applied
//    to the fp32 result. Exact for every group whose exponent is within 36
//    binades of its row's largest (smaller groups lose low bits).
//  * Activations are staged as f16 in shared memory, bf16 inputs scaled per
//    token by a power of two that puts the row maximum in [2^14, 2^15) (exact
//    for every element within 2^-29 of the row maximum), in the K order that
//    makes each lane's 16-byte weight load feed eight m16n8k16 steps.
//  * mma.sync m16n8k16 with fp32 accumulation; the 8 warps split K and their
//    partial tiles are summed in a fixed order through shared memory.
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.cuh"
#include "ptx.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kDW = 8;                 // warps per CTA
constexpr int kDThreads = kDW * 32;
constexpr int kTileRows = 16;          // weight rows per tile (one m16 MMA tile)
constexpr int kChunk = 16;             // tokens staged at once in k_dec_w2 (two n8 tiles)
constexpr int kChunk13 = 8;            // tokens staged at once in k_dec_w13 (one n8 tile)
constexpr int kStages = 3;             // weight tiles in flight per CTA (k_dec_w2)
constexpr uint32_t kWaitTries = 1u << 20;

enum { kMx = 0, kS8 = 1 };

struct DecParams {
  int T, H, I, Is, E, k;
  float limit;
  const __nv_bfloat16* x;
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
  __half* h;    // [T*k, I] routed intermediates, sorted-slot order
  __half* hs;   // [T, I_s] shared intermediates
  __nv_bfloat16* out;
  uint32_t* status;
};

// Row layout of a weight tile in shared memory: 16 rows, padded so that the
// 8-lane phases of 16-byte reads touch distinct banks.
__host__ __device__ inline int tile_stride(int fmt, int K) {
  const int rb = fmt == kMx ? K / 2 : K;
  return fmt == kMx ? rb + ((rb % 128 == 0) ? 64 : 0) : rb + 16;
}
__host__ __device__ inline int tile_bytes(int fmt, int K) { return kTileRows * tile_stride(fmt, K); }
__host__ __device__ inline int xs_stride(int K) { return K * 2 + 16; }

// Logical (MMA) position of physical element e within a 128-element block:
// lane t of a quad owns physical [32t, 32t+32); step s of the block uses its
// elements 4s..4s+3 at logical columns {2t, 2t+1, 2t+8, 2t+9}.
__device__ __forceinline__ int logical_pair_offset(int e_pair0) {
  // e_pair0: physical index (even) of an element pair inside the block
  const int t = e_pair0 >> 5, q = e_pair0 & 31;
  const int s = q >> 2, c = q & 3;  // c is 0 or 2
  return s * 16 + (c ? 8 : 0) + 2 * t;
}

// Stage `n` activation rows into xs (f16, logical order). Rows come from
// bf16 `x` (per-row power-of-two scaling, exponent stored in sigma[]) or from
// f16 `hsrc` (no scaling). Row r of the chunk is source row row_of(r).
template <bool FROM_BF16>
__device__ void stage_rows(char* xs, int K, int n, const void* src, const int32_t* row_map, int row_base,
                           int kdiv, int* sigma) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int xstr = xs_stride(K);
  for (int r = warp; r < n; r += kDW) {
    const int row = row_map ? __ldg(row_map + row_base + r) / kdiv : row_base + r;
    const uint4* s4 = reinterpret_cast<const uint4*>(static_cast<const char*>(src) + size_t(row) * K * 2);
    char* dst = xs + size_t(r) * xstr;
    float mul = 1.0f;
    if (FROM_BF16) {
      uint32_t mx = 0;
      for (int p = lane; p < K / 8; p += 32) {
        const uint4 v = __ldg(s4 + p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) mx = max(mx, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      // bf16 bits without sign: exponent field in bits 14..7
      const int ef = int(mx >> 7);
      int sg = (mx == 0 || ef == 0) ? 0 : 141 - ef;  // 14 - floor(log2(max))
      if (mx != 0 && ef == 0) sg = 120;               // bf16 subnormal maximum
      sg = max(-120, min(120, sg));
      if (lane == 0) sigma[r] = sg;
      mul = __int_as_float((sg + 127) << 23);
    }
    for (int p = lane; p < K / 8; p += 32) {
      const uint4 v = __ldg(s4 + p);
      const int e0 = p * 8;
      const int blk = e0 >> 7, within = e0 & 127;
      uint32_t w[4];
      if (FROM_BF16) {
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __half2 hv = __floats2half2_rn(bf16_lo(in[i]) * mul, bf16_hi(in[i]) * mul);
          w[i] = *reinterpret_cast<const uint32_t*>(&hv);
        }
      } else {
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int L = blk * 128 + logical_pair_offset(within + 2 * i);
        *reinterpret_cast<uint32_t*>(dst + L * 2) = w[i];
      }
    }
  }
}

// Issue the bulk copies of a 16-row weight tile (row i of the tile is global
// row rows[i]) and arm `bar` with the byte count. Called by one thread.
__device__ __forceinline__ void load_tile(char* wt, int wstride, const uint8_t* base, const int* rows,
                                          int rowbytes, uint64_t* bar) {
  mbar_arrive_expect_tx(bar, uint32_t(kTileRows * rowbytes));
#pragma unroll 1
  for (int i = 0; i < kTileRows; ++i)
    bulk_g2s(wt + i * wstride, base + size_t(rows[i]) * rowbytes, uint32_t(rowbytes), bar);
}

// Per-row largest E8M0 exponent of a 16-row tile (rows given by rows[]) into
// rowx[16]; the per-(row, group) f16 operand scales are derived from it.
__device__ __forceinline__ void tile_row_max_exp(const uint8_t* scales, const int* rows, int K, int* rowx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = K / 32;
  for (int r = warp; r < kTileRows; r += kDW) {
    const uint8_t* sr = scales + size_t(rows[r]) * G;
    int m = 0;
    for (int g = lane; g < G; g += 32) m = max(m, int(__ldg(sr + g)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) rowx[r] = m;
  }
}

// One warp's share of a 16-row tile times the staged activation rows: K
// blocks blk = warp, warp + kDW, ... Accumulates into acc[NT][4] (fp32 C
// fragments, rows (g, g+8), token columns (2t, 2t+1) of each n8 tile).
template <int FMT, int NT>
__device__ __forceinline__ void warp_tile_mma(const char* wt, int wstride, const char* xs, int K, int nrows,
                                              const uint8_t* scales, const int* rows, const int* rowx,
                                              float acc[NT][4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int xstr = xs_stride(K);
  const int nblk = K / 128;
  // ldmatrix source rows (token = lane & 7 within each n8 tile, clamped to the chunk)
  uint32_t xaddr[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    int tok = nt * 8 + (lane & 7);
    tok = min(tok, nrows - 1);
    xaddr[nt] = smem_u32(xs + size_t(tok) * xstr) + ((lane >> 3) & 1) * 16 + (lane >> 4) * 32;
  }
  const uint8_t* srow_a = nullptr;
  const uint8_t* srow_b = nullptr;
  int xa = 0, xb = 0;
  if (FMT == kMx) {
    srow_a = scales + size_t(rows[g]) * (K / 32);
    srow_b = scales + size_t(rows[g + 8]) * (K / 32);
    xa = rowx[g];
    xb = rowx[g + 8];
  }
  for (int b = warp; b < nblk; b += kDW) {
    uint32_t A[8][4];  // per step s: a0..a3
    if (FMT == kMx) {
      const uint4 qa = *reinterpret_cast<const uint4*>(wt + g * wstride + b * 64 + 16 * t);
      const uint4 qb = *reinterpret_cast<const uint4*>(wt + (g + 8) * wstride + b * 64 + 16 * t);
      const uint32_t sa = f16_pow2_bits(int(__ldg(srow_a + 4 * b + t)) - xa + 13) * 0x10001u;
      const uint32_t sb = f16_pow2_bits(int(__ldg(srow_b + 4 * b + t)) - xb + 13) * 0x10001u;
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
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(b0, b1, b2, b3, xaddr[nt] + (b * 128 + sp * 32) * 2);
        mma_16816_f16(acc[nt], A[2 * sp], b0, b1);
        mma_16816_f16(acc[nt], A[2 * sp + 1], b2, b3);
      }
    }
  }
}

// Sum the 8 warps' C fragments in warp order; result valid in warp 0.
template <int NT>
__device__ __forceinline__ void reduce_warps(float acc[NT][4], float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[((warp * NT + nt) * 4 + i) * 32 + lane] = acc[nt][i];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s = 0.f;
        for (int w = 0; w < kDW; ++w) s += red[((w * NT + nt) * 4 + i) * 32 + lane];
        acc[nt][i] = s;
      }
  }
}

__device__ __forceinline__ bool wait_tile(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_wait_bounded(bar, parity, kWaitTries)) return true;
  if (threadIdx.x == 0) atomicOr(status, kStatusTimeout);
  // the copies target this CTA's shared memory: wait for them before leaving
  mbar_wait_bounded(bar, parity, kWaitTries << 4);
  return false;
}

__device__ __forceinline__ float pow2f(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((e + 127) << 23);
}

// Compact list of non-empty groups in ascending order (routed experts, then
// the shared expert as group E): list[0..*n). One warp, ballot compaction.
__device__ __forceinline__ void build_hit_list(const int32_t* offsets, int E, bool has_shared, int* list,
                                               int* n_out) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int n = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const bool hit = e < E && __ldg(offsets + e + 1) > __ldg(offsets + e);
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      if (hit) list[n + __popc(m & ((1u << lane) - 1u))] = e;
      n += __popc(m);
    }
    if (lane == 0) {
      if (has_shared) list[n++] = E;
      *n_out = n;
    }
  }
}

// ------------------------------------------------------------------ w13

// Persistent over work items (group, 8-channel block): routed hit experts in
// ascending id with I/8 blocks each, then the shared expert with I_s/8. Each
// CTA takes a contiguous range of items (so staged activations are reused
// while the group does not change) and double-buffers the weight tiles.
constexpr int kW13Stages = 2;

struct W13Item {
  int grp, j0;
};

__global__ void __launch_bounds__(kDThreads) k_dec_w13(DecParams P, int stage_bytes) {
  extern __shared__ __align__(128) char smem[];
  const int H = P.H;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);          // [kW13Stages]
  int* rows = reinterpret_cast<int*>(smem + 64);                 // [kW13Stages][16]
  int* rowx = rows + kW13Stages * 16;                            // [kW13Stages][16]
  int* sigma = rowx + kW13Stages * 16;                           // [kChunk13]
  int* nlist = sigma + kChunk;                                   // [1]
  int* list = reinterpret_cast<int*>(smem + 512);                // [E + 1]
  float* red = reinterpret_cast<float*>(smem + 512 + ((P.E + 1) * 4 + 127) / 128 * 128);  // [kDW][4][32]
  char* wts = reinterpret_cast<char*>(red + kDW * 4 * 32);
  char* xs = wts + size_t(kW13Stages) * stage_bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kW13Stages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  pdl_wait();  // offsets / sorted_slot come from the permutation kernel
  build_hit_list(P.offsets, P.E, P.Is > 0, list, nlist);
  __syncthreads();
  const int nl = *nlist;
  const bool has_shared = P.Is > 0;
  const int n_routed = has_shared ? nl - 1 : nl;
  const int blk_r = P.I / 8, blk_s = P.Is / 8;
  const int n_items = n_routed * blk_r + (has_shared ? blk_s : 0);
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per, it1 = min(n_items, it0 + per);
  if (it0 >= it1) return;
  auto item = [&](int it) {
    W13Item w;
    if (it < n_routed * blk_r) {
      w.grp = list[it / blk_r];
      w.j0 = (it % blk_r) * 8;
    } else {
      w.grp = P.E;
      w.j0 = (it - n_routed * blk_r) * 8;
    }
    return w;
  };
  auto issue = [&](int it, int s) {  // thread 0 only
    const W13Item w = item(it);
    const bool sh = w.grp == P.E;
    const int Ig = sh ? P.Is : P.I;
    int* r = rows + s * 16;
    for (int i = 0; i < kTileRows; ++i) r[i] = i < 8 ? w.j0 + i : Ig + w.j0 + (i - 8);
    const uint8_t* base = sh ? reinterpret_cast<const uint8_t*>(P.sh13)
                             : P.w13_codes + size_t(w.grp) * 2 * P.I * (H / 2);
    load_tile(wts + size_t(s) * stage_bytes, tile_stride(sh ? kS8 : kMx, H), base, r, sh ? H : H / 2,
              &bars[s]);
  };
  if (threadIdx.x == 0)
    for (int s = 0; s < kW13Stages && it0 + s < it1; ++s) issue(it0 + s, s);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  int staged_grp = -1, staged_chunk = -1;
  for (int it = it0; it < it1; ++it) {
    const int i = it - it0;
    const int s = i % kW13Stages;
    const uint32_t parity = uint32_t(i / kW13Stages) & 1u;
    const W13Item w = item(it);
    const bool sh = w.grp == P.E;
    const int fmt = sh ? kS8 : kMx;
    const int Ig = sh ? P.Is : P.I;
    const int r0 = sh ? 0 : P.offsets[w.grp];
    const int nrows = sh ? P.T : P.offsets[w.grp + 1] - r0;
    const uint8_t* sbase = sh ? nullptr : P.w13_scales + size_t(w.grp) * 2 * P.I * (H / 32);
    if (fmt == kMx) tile_row_max_exp(sbase, rows + s * 16, H, rowx + s * 16);
    if (!wait_tile(&bars[s], parity, P.status)) {
      // give the other copies in flight (later items) a bounded wait, then leave
      for (int q = 1; q < kW13Stages && it + q < it1; ++q)
        mbar_wait_bounded(&bars[(i + q) % kW13Stages], uint32_t((i + q) / kW13Stages) & 1u, kWaitTries);
      return;
    }
    const char* wt = wts + size_t(s) * stage_bytes;
    for (int c = 0; c < nrows; c += kChunk13) {
      const int n = min(kChunk13, nrows - c);
      if (staged_grp != w.grp || staged_chunk != c) {
        __syncthreads();  // readers of the previous staging are done
        stage_rows<true>(xs, H, n, P.x, sh ? nullptr : P.sorted_slot, r0 + c, P.k, sigma);
        staged_grp = w.grp;
        staged_chunk = c;
      }
      __syncthreads();
      float acc[1][4] = {};
      if (fmt == kMx)
        warp_tile_mma<kMx, 1>(wt, tile_stride(kMx, H), xs, H, n, sbase, rows + s * 16, rowx + s * 16, acc);
      else
        warp_tile_mma<kS8, 1>(wt, tile_stride(kS8, H), xs, H, n, nullptr, rows + s * 16, rowx + s * 16, acc);
      reduce_warps<1>(acc, red);
      if (warp == 0) {
        float fg, fu;
        if (fmt == kMx) {
          fg = pow2f(rowx[s * 16 + g] - 127 - 13);
          fu = pow2f(rowx[s * 16 + g + 8] - 127 - 13);
        } else {
          fg = __ldg(P.sh13_scale + w.j0 + g);
          fu = __ldg(P.sh13_scale + Ig + w.j0 + g);
        }
        __half* hout = sh ? P.hs : P.h;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int nn = 2 * t + q;
          if (nn < n) {
            const float inv = pow2f(-sigma[nn]);
            const float gv = acc[0][q] * fg * inv;
            const float uv = acc[0][2 + q] * fu * inv;
            hout[size_t(r0 + c + nn) * Ig + w.j0 + g] = __float2half_rn(clamped_swiglu_f(gv, uv, P.limit));
          }
        }
      }
    }
    __syncthreads();  // every warp is done with stage s (and with rows/rowx of s)
    if (threadIdx.x == 0 && it + kW13Stages < it1) issue(it + kW13Stages, s);
  }
}

// ------------------------------------------------------------------ w2 + combine

template <int NT>
__global__ void __launch_bounds__(kDThreads) k_dec_w2(DecParams P, int stage_bytes) {
  extern __shared__ __align__(128) char smem[];
  const int H = P.H;
  const int m0 = blockIdx.x * kTileRows;
  const int T = P.T;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);               // [kStages]
  int* rows = reinterpret_cast<int*>(smem + 64);                     // [16]
  int* rowx = rows + 16;                                             // [16]
  int* nlist = rowx + 16;                                            // [1]
  int* list = reinterpret_cast<int*>(smem + 512);                    // [E + 1]
  float* red = reinterpret_cast<float*>(smem + 512 + ((P.E + 1) * 4 + 127) / 128 * 128);  // [kDW][NT][4][32]
  float* oacc = red + kDW * NT * 4 * 32;                             // [T][16]
  char* wts = reinterpret_cast<char*>(oacc + size_t(T) * kTileRows);
  wts = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(wts) + 127) & ~uintptr_t(127));
  char* xs = wts + size_t(kStages) * stage_bytes;

  if (threadIdx.x < kTileRows) rows[threadIdx.x] = m0 + threadIdx.x;
  for (int i = threadIdx.x; i < T * kTileRows; i += kDThreads) oacc[i] = 0.f;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  pdl_wait();  // h (all groups) and the routing come from the previous kernels
  build_hit_list(P.offsets, P.E, P.Is > 0, list, nlist);
  __syncthreads();
  const int nl = *nlist;
  auto issue = [&](int li, int s) {  // thread 0 only
    const int gi = list[li];
    const bool sh = gi == P.E;
    const int Kg = sh ? P.Is : P.I;
    const uint8_t* base = sh ? reinterpret_cast<const uint8_t*>(P.sh2) : P.w2_codes + size_t(gi) * H * (P.I / 2);
    load_tile(wts + size_t(s) * stage_bytes, tile_stride(sh ? kS8 : kMx, Kg), base, rows, sh ? Kg : Kg / 2,
              &bars[s]);
  };
  if (threadIdx.x == 0)
    for (int s = 0; s < kStages && s < nl; ++s) issue(s, s);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  for (int li = 0; li < nl; ++li) {
    const int s = li % kStages;
    const uint32_t parity = uint32_t(li / kStages) & 1u;
    const int gi = list[li];
    const bool sh = gi == P.E;
    const int fmt = sh ? kS8 : kMx;
    const int Kg = sh ? P.Is : P.I;
    const int r0 = sh ? 0 : P.offsets[gi];
    const int n = sh ? T : P.offsets[gi + 1] - r0;
    const uint8_t* sbase = sh ? nullptr : P.w2_scales + size_t(gi) * H * (P.I / 32);
    if (fmt == kMx) tile_row_max_exp(sbase, rows, Kg, rowx);
    if (!wait_tile(&bars[s], parity, P.status)) {
      for (int q = 1; q < kStages && li + q < nl; ++q)
        mbar_wait_bounded(&bars[(li + q) % kStages], uint32_t((li + q) / kStages) & 1u, kWaitTries);
      return;
    }
    const char* wt = wts + size_t(s) * stage_bytes;
    for (int c = 0; c < n; c += kChunk) {
      const int nc = min(kChunk, n - c);
      __syncthreads();
      stage_rows<false>(xs, Kg, nc, sh ? static_cast<const void*>(P.hs) : static_cast<const void*>(P.h),
                        nullptr, r0 + c, 1, nullptr);
      __syncthreads();
      float acc[NT][4] = {};
      if (fmt == kMx)
        warp_tile_mma<kMx, NT>(wt, tile_stride(kMx, Kg), xs, Kg, nc, sbase, rows, rowx, acc);
      else
        warp_tile_mma<kS8, NT>(wt, tile_stride(kS8, Kg), xs, Kg, nc, nullptr, rows, rowx, acc);
      reduce_warps<NT>(acc, red);
      if (warp == 0) {
        float fa, fb;
        if (fmt == kMx) {
          fa = pow2f(rowx[g] - 127 - 13);
          fb = pow2f(rowx[g + 8] - 127 - 13);
        } else {
          fa = __ldg(P.sh2_scale + m0 + g);
          fb = __ldg(P.sh2_scale + m0 + g + 8);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int nn = nt * 8 + 2 * t + q;
            if (nn < nc) {
              int tok;
              float wgt;
              if (sh) {
                tok = r0 + c + nn;
                wgt = 1.0f;
              } else {
                const int slot = __ldg(P.sorted_slot + r0 + c + nn);
                tok = slot / P.k;
                wgt = __ldg(P.topk_w + slot);
              }
              atomicAdd(&oacc[tok * kTileRows + g], wgt * (acc[nt][q] * fa));
              atomicAdd(&oacc[tok * kTileRows + g + 8], wgt * (acc[nt][2 + q] * fb));
            }
          }
      }
    }
    __syncthreads();  // every warp is done with stage s and rowx
    if (threadIdx.x == 0 && li + kStages < nl) issue(li + kStages, s);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < T * kTileRows; i += kDThreads) {
    const int tok = i / kTileRows, r = i % kTileRows;
    P.out[size_t(tok) * H + m0 + r] = __float2bfloat16_rn(oacc[i]);
  }
}

}  // namespace

static int w13_stage_bytes(const v4moe_config& c) {
  return std::max(tile_bytes(kMx, c.hidden), c.shared_inter > 0 ? tile_bytes(kS8, c.hidden) : 0);
}
static int w2_stage_bytes(const v4moe_config& c) {
  return std::max(tile_bytes(kMx, c.inter), c.shared_inter > 0 ? tile_bytes(kS8, c.shared_inter) : 0);
}
static size_t list_bytes(const v4moe_config& c) { return size_t((c.n_experts + 1) * 4 + 127) / 128 * 128; }

size_t dec_w13_smem(const v4moe_config& c, int T) {
  const int chunk = T < kChunk13 ? T : kChunk13;
  return 512 + list_bytes(c) + size_t(kDW) * 4 * 32 * 4 + size_t(kW13Stages) * w13_stage_bytes(c) +
         size_t(chunk) * xs_stride(c.hidden);
}

size_t dec_w2_smem(const v4moe_config& c, int T, int NT) {
  const int chunk = T < kChunk ? T : kChunk;
  const int K = std::max(c.inter, c.shared_inter);
  return 512 + list_bytes(c) + size_t(kDW) * NT * 4 * 32 * 4 + size_t(T) * kTileRows * 4 + 128 +
         size_t(kStages) * w2_stage_bytes(c) + size_t(chunk) * xs_stride(K);
}

bool dec_supported(const v4moe_config& c, int T) {
  return T <= kDecodeMaxTokens && dec_w13_smem(c, T) <= 227 * 1024 && dec_w2_smem(c, T, 2) <= 227 * 1024;
}

cudaError_t launch_forward_dec(const ForwardArgs& a, cudaStream_t st) {
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
  P.x = a.x;
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
  P.h = reinterpret_cast<__half*>(a.h);
  P.hs = reinterpret_cast<__half*>(a.hs);
  P.out = a.out;
  P.status = a.status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t s13 = dec_w13_smem(c, a.T);
  set_smem(k_dec_w13, s13);
  int occ = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_dec_w13, kDThreads, s13);
  occ = std::max(1, occ);
  cudaError_t e = launch_kernel("dec_w13", k_dec_w13, dim3(sms * occ), dim3(kDThreads), s13, st, true, P,
                                w13_stage_bytes(c));
  if (e != cudaSuccess) return e;
  if (a.T > 8) {
    const size_t s2 = dec_w2_smem(c, a.T, 2);
    set_smem(k_dec_w2<2>, s2);
    return launch_kernel("dec_w2", k_dec_w2<2>, dim3(c.hidden / kTileRows), dim3(kDThreads), s2, st, true, P,
                         w2_stage_bytes(c));
  }
  const size_t s2 = dec_w2_smem(c, a.T, 1);
  set_smem(k_dec_w2<1>, s2);
  return launch_kernel("dec_w2", k_dec_w2<1>, dim3(c.hidden / kTileRows), dim3(kDThreads), s2, st, true, P,
                       w2_stage_bytes(c));
}

}  // namespace v4moe
