// Shared expert on tcgen05 for large batches: a token-major f16 GEMM fed by
// TMA on both operands, with the combine of the routed outputs fused into the
// down projection's epilogue.
//
// What it computes ("Checked in its code" rows "Shared expert" and "SwiGLU
// feed-forward"; "config.json" linears_w8a16: int8, symmetric, one scale per
// output channel):
//   w13: hs[t, c] = silu(min(s_g[c] g, L)) * clamp(s_u[c] u, -L, L),
//        g = q13[c] . x_t, u = q13[Is + c] . x_t                     (f16 out)
//   w2:  out[t, m] = bf16( sum_j w[t, j] y_slot[slot(t, j), m] + s2[m] (q2[m] . hs_t) )  (y_slot bf16)
// with the routed expert outputs y_slot of the same call, summed in slot order
// j = 0 .. k-1 and then the shared term, so the result does not depend on
// timing.
//
// Operands: the int8 weights are first widened to f16 in the workspace
// (exact: |q| <= 127), so the GEMM reads both operands by TMA with no
// dequantisation in the loop; the activations are the f16 copy of x scaled
// per token by 2^sigma (exact), undone in the epilogue, and the f16
// intermediates hs.
//
// Tile: 128 tokens (MMA M) x 256 weight rows (MMA N); w13 tiles take 128 gate
// rows and the matching 128 up rows, so the SwiGLU pairs sit in one thread.
// One persistent CTA per SM:
//   warp 0      TMA producer (4 stages of 64 K: 16 KB activations, 32 KB weights)
//   warp 1      TMEM owner and tcgen05.mma issuer (kind::f16, fp32 accumulate)
//   warps 2-9   epilogue, two per TMEM lane quarter (warp % 4), each half of
//               the 256 accumulator columns in rounds of 32; the w2 epilogue
//               transposes the shared term through shared memory and reads
//               the routed rows four tokens per load instruction
// The fp32 accumulator (128 lanes x 256 columns) is double-buffered in TMEM,
// so a tile's epilogue overlaps the next tile's MMAs.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>

#include "launch.cuh"
#include "ptx.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int SMt = 128;   // tokens per tile
constexpr int SNr = 256;   // weight rows per tile
constexpr int SKc = 64;    // K per stage
constexpr int kSStages = 4;
constexpr int kSFirstEpi = 2;
constexpr int kSEpiWarps = 8;
constexpr int kSThreads = 32 * (kSFirstEpi + kSEpiWarps);
constexpr int kSA = SMt * SKc * 2;   // 16 KB
constexpr int kSB = SNr * SKc * 2;   // 32 KB
constexpr int kSStage = kSA + kSB;
constexpr int kSXch = 33;    // transpose buffer row stride (floats)
constexpr int kSOffX = kSStages * kSStage;                  // [8 warps][32][33] fp32
constexpr int kSOffBar = kSOffX + kSEpiWarps * 32 * kSXch * 4;
constexpr int kSSmem = kSOffBar + 256 + 1024;
static_assert(kSSmem <= 232448, "dynamic shared memory per block");
constexpr uint32_t kSTries = 1u << 21;

enum { kSW13 = 0, kSW2 = 1, kSLin = 2 };

struct SBars {
  uint64_t full[kSStages];
  uint64_t empty[kSStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SBars) <= 256, "barrier block");

struct ShParams {
  int T, H, Is, E, k;
  float limit;
  int mode;
  int nb;      // weight-row blocks per token tile
  int ntiles;  // token tiles x nb
  int nk;      // K chunks
  const int* sigma;      // [T] exponents of the f16 activations (w13)
  const float* scale;    // w13: [2 Is] row scales; w2: [H]
  __half* hs;            // w13 out [T, Is]
  const int32_t* topk_ids;
  const float* topk_w;
  const int32_t* slot_pos;
  const __nv_bfloat16* y_slot;  // [T k, H] routed outputs in slot order (bf16)
  __nv_bfloat16* out;    // [T, H]; linear mode: [T, G N]
  // linear mode: G groups of N output channels over K inputs each (group g
  // reads x columns g K .. and weight rows g N ..); bn weight rows per tile
  // (128 or 256, nbg blocks per group); order 1 walks the token tiles of a
  // weight block before the next block (mt token tiles).
  int G, N, K, bn, nbg, mt, order;
  uint32_t* status;
};

// Tile ti -> first token, weight-row block (over all groups in linear mode).
__device__ __forceinline__ void tile_of(const ShParams& P, int ti, int& t0, int& rb) {
  if (P.order) {
    rb = ti / P.mt;
    t0 = (ti - rb * P.mt) * SMt;
  } else {
    t0 = (ti / P.nb) * SMt;
    rb = ti % P.nb;
  }
}

__device__ __forceinline__ bool swait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  for (uint32_t i = 0; i < kSTries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
  return false;
}

__device__ __forceinline__ void tma_load_3d_s(void* dst, const void* tmap, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((max(-126, min(127, e)) + 127) << 23); }

// One round of the combine (32 output rows from m0) for a warp's 32 tokens
// (first token tq): lane l takes token 4 g + l / 8 and columns 4 (l % 8) .. + 3
// for g = 0 .. 7, so a load instruction reads four tokens' 128-byte row
// pieces; all of a token's NJ slot rows are in flight at once (slots that do
// not exist read row 0 and are left out of the sum). wj / pj: this lane's
// token's routing weights and slot positions; tb: the shared term of the
// round, [token][column] with row stride kSXch.
template <int NJ>
__device__ __forceinline__ void combine_round(const ShParams& P, const float (&wj)[8], const int (&pj)[8],
                                              const float* tb, int tq, int sl, int c4, int m0) {
#pragma unroll 2
  for (int g = 0; g < 8; ++g) {
    const int tl = 4 * g + sl;  // token within the warp's 32
    float w[NJ];
    int p[NJ];
    uint2 y[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      w[j] = __shfl_sync(0xffffffffu, wj[j], tl);
      p[j] = __shfl_sync(0xffffffffu, pj[j], tl);
      y[j] = __ldg(reinterpret_cast<const uint2*>(P.y_slot + size_t(max(p[j], 0)) * P.H + m0 + c4));
    }
    float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      if (p[j] >= 0) {
        a.x = fmaf(w[j], __uint_as_float(y[j].x << 16), a.x);
        a.y = fmaf(w[j], __uint_as_float(y[j].x & 0xFFFF0000u), a.y);
        a.z = fmaf(w[j], __uint_as_float(y[j].y << 16), a.z);
        a.w = fmaf(w[j], __uint_as_float(y[j].y & 0xFFFF0000u), a.w);
      }
    }
    const int t2 = tq + tl;
    if (t2 < P.T) {
      const float* sp = tb + tl * kSXch + c4;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x + sp[0], a.y + sp[1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(a.z + sp[2], a.w + sp[3]);
      *reinterpret_cast<uint2*>(P.out + size_t(t2) * P.H + m0 + c4) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
}

__global__ void __launch_bounds__(kSThreads, 1)
    k_sh_gemm(ShParams P, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SBars& B = *reinterpret_cast<SBars*>(smem + kSOffBar);
  volatile int* abort_flag = &B.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool w13 = P.mode == kSW13;
  const bool lin = P.mode == kSLin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&B.full[s], 1);
      mbar_init(&B.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.acc_full[b], 1);
      mbar_init(&B.acc_empty[b], kSEpiWarps);
    }
    mbar_init(&B.done, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&B.tmem_base, 2 * SNr);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;
  pdl_wait();  // activations, widened weights and routed outputs come from earlier kernels

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    uint32_t gc = 0;
    bool ok = true;
    const uint32_t stage_bytes = uint32_t(kSA + (lin ? P.bn : SNr) * SKc * 2);
    for (int ti = blockIdx.x; ti < P.ntiles && ok; ti += gridDim.x) {
      int t0, rb;
      tile_of(P, ti, t0, rb);
      const int g = lin ? rb / P.nbg : 0;
      const int acol = lin ? g * P.K : 0;
      const int brow = lin ? g * P.N + (rb - g * P.nbg) * P.bn : rb * SNr;
      for (int c = 0; c < P.nk; ++c, ++gc) {
        const int s = gc % kSStages;
        const uint32_t u = gc / kSStages;
        if (!swait(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        char* st = smem + s * kSStage;
        mbar_arrive_expect_tx(&B.full[s], stage_bytes);
        tma_load_2d(st, &tmA, acol + c * SKc, t0, &B.full[s]);
        if (w13)  // 128 gate rows, then the matching 128 up rows
          tma_load_3d_s(st + kSA, &tmB, c * SKc, rb * (SNr / 2), 0, &B.full[s]);
        else
          tma_load_2d(st + kSA, &tmB, c * SKc, brow, &B.full[s]);
      }
    }
    // nothing may still be landing in shared memory when the CTA exits
    for (uint32_t q = 0; q < uint32_t(kSStages) && q < gc; ++q) {
      const uint32_t gq = gc - 1 - q;
      mbar_wait_bounded(&B.full[gq % kSStages], (gq / kSStages) & 1u, kSTries);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t gc = 0, lt = 0;
    bool ok = true;
    const uint32_t idesc = lin ? idesc_bf16_f32(SMt, P.bn) : idesc_f16_f32(SMt, SNr);
    for (int ti = blockIdx.x; ti < P.ntiles && ok; ti += gridDim.x, ++lt) {
      const uint32_t b = lt & 1u, v = lt >> 1;
      if (!swait(&B.acc_empty[b], (v & 1u) ^ 1u, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t d = tmem + b * SNr;
      for (int c = 0; c < P.nk; ++c, ++gc) {
        const int s = gc % kSStages;
        const uint32_t u = gc / kSStages;
        if (!swait(&B.full[s], u & 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * kSStage);
        const uint32_t b0 = a0 + kSA;
#pragma unroll
        for (int kk = 0; kk < SKc / 16; ++kk)
          umma_f16_ss(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                      (c > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&B.empty[s]);
      }
      if (!ok) break;
      umma_commit(&B.acc_full[b]);
    }
    umma_commit(&B.done);
    mbar_wait_bounded(&B.done, 0, kSTries);
  } else if (warp >= kSFirstEpi) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quarter
    const int half = (warp - kSFirstEpi) >> 2;  // half of the columns
    uint32_t lt = 0;
    for (int ti = blockIdx.x; ti < P.ntiles; ti += gridDim.x, ++lt) {
      const uint32_t b = lt & 1u, v = lt >> 1;
      int t0, rb;
      tile_of(P, ti, t0, rb);
      if (!__all_sync(0xffffffffu, swait(&B.acc_full[b], v & 1u, abort_flag, P.status)) || *abort_flag) break;
      tc_fence_after();
      const uint32_t acc = tmem + b * SNr + (uint32_t(32 * q) << 16);
      if (lin) {
        // out[t, g N + n] = bf16(scale[g N + n] * acc): bn / 2 channels per
        // warp in rounds of 32
        const int t = t0 + 32 * q + lane;
        const int g = rb / P.nbg;
        const int nrounds = P.bn / 64;
        const size_t ld = size_t(P.G) * P.N;
#pragma unroll 1
        for (int r = 0; r < nrounds; ++r) {
          const int cc = (P.bn / 2) * half + 32 * r;
          uint32_t ra[32];
          tmem_ld_32x32b_x32(acc + cc, ra);
          tmem_wait_ld();
          if (r == nrounds - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.acc_empty[b]);
          }
          const int nl = (rb - g * P.nbg) * P.bn + cc;  // channel within the group
          if (t < P.T && nl < P.N) {  // N % 32 == 0: a round is all in or all out
            const int n0 = g * P.N + nl;
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(ra[i]) * __ldg(P.scale + n0 + i),
                                                             __uint_as_float(ra[i + 1]) * __ldg(P.scale + n0 + i + 1));
              o[i >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(P.out + size_t(t) * ld + n0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
        }
        continue;
      }
      const int tok = t0 + 32 * q + lane;
      const bool valid = tok < P.T;
      if (w13) {
        // 64 channels in two rounds: gate columns c, up columns 128 + c
        const float inv = valid ? pow2i(-P.sigma[tok]) : 0.0f;
#pragma unroll 1
        for (int r = 0; r < 2; ++r) {
          const int cc = 64 * half + 32 * r;  // column within the 128 channels
          uint32_t ga[32], ua[32];
          tmem_ld_32x32b_x32(acc + cc, ga);
          tmem_ld_32x32b_x32(acc + SNr / 2 + cc, ua);
          tmem_wait_ld();
          if (r == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.acc_empty[b]);
          }
          const int c0 = rb * (SNr / 2) + cc;
          if (valid) {
            uint32_t hw[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float g0 = __uint_as_float(ga[i]) * __ldg(P.scale + c0 + i) * inv;
              const float g1 = __uint_as_float(ga[i + 1]) * __ldg(P.scale + c0 + i + 1) * inv;
              const float u0 = __uint_as_float(ua[i]) * __ldg(P.scale + P.Is + c0 + i) * inv;
              const float u1 = __uint_as_float(ua[i + 1]) * __ldg(P.scale + P.Is + c0 + i + 1) * inv;
              const __half2 h =
                  __floats2half2_rn(clamped_swiglu_f(g0, u0, P.limit), clamped_swiglu_f(g1, u1, P.limit));
              hw[i >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(P.hs + size_t(tok) * P.Is + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(hw[4 * i], hw[4 * i + 1], hw[4 * i + 2], hw[4 * i + 3]);
          }
        }
      } else {
        // combine, 128 output rows in four rounds of 32: the shared term
        // (thread = token) goes through this warp's transpose buffer, then
        // combine_round adds the routed slots.
        float wj[8];
        int pj[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          wj[j] = 0.0f;
          pj[j] = -1;
          if (valid && j < P.k) {
            const int e = P.topk_ids[size_t(tok) * P.k + j];
            if (e >= 0 && e < P.E) {
              wj[j] = P.topk_w[size_t(tok) * P.k + j];
              pj[j] = P.slot_pos[size_t(tok) * P.k + j];
            }
          }
        }
        float* tb = reinterpret_cast<float*>(smem + kSOffX) + (warp - kSFirstEpi) * 32 * kSXch;
        const int sl = lane >> 3, c4 = (lane & 7) * 4;
#pragma unroll 1
        for (int r = 0; r < 4; ++r) {
          const int cc = 128 * half + 32 * r;
          const int m0 = rb * SNr + cc;
          uint32_t ra[32];
          tmem_ld_32x32b_x32(acc + cc, ra);
          tmem_wait_ld();
          if (r == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.acc_empty[b]);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) tb[lane * kSXch + i] = __uint_as_float(ra[i]) * __ldg(P.scale + m0 + i);
          __syncwarp();
          if (P.k <= 6)
            combine_round<6>(P, wj, pj, tb, t0 + 32 * q, sl, c4, m0);
          else
            combine_round<8>(P, wj, pj, tb, t0 + 32 * q, sl, c4, m0);
          __syncwarp();
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * SNr);
  }
}

// int8 -> f16, exact; n % 16 == 0, both pointers 16-byte aligned. Each thread
// converts four 16-byte pieces per pass with all four loads in flight.
__global__ void __launch_bounds__(256) k_s8_to_f16(const int8_t* __restrict__ a, __half* __restrict__ fa, size_t na,
                                                   const int8_t* __restrict__ b, __half* __restrict__ fb, size_t nb) {
  pdl_wait();  // the previous call's kernels may still read the widened copies
  const size_t n16a = na / 16, n16 = n16a + nb / 16;
  const size_t step = size_t(gridDim.x) * blockDim.x;
  for (size_t i0 = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i0 < n16; i0 += 4 * step) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t i = i0 + u * step;
      if (i < n16) q[u] = __ldg(reinterpret_cast<const uint4*>(i < n16a ? a : b) + (i < n16a ? i : i - n16a));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t i = i0 + u * step;
      if (i >= n16) break;
      const bool first = i < n16a;
      const size_t j = first ? i : i - n16a;
      uint4 lo, hi;
      s8x4_to_f16x2(q[u].x, lo.x, lo.y);
      s8x4_to_f16x2(q[u].y, lo.z, lo.w);
      s8x4_to_f16x2(q[u].z, hi.x, hi.y);
      s8x4_to_f16x2(q[u].w, hi.z, hi.w);
      uint4* d = reinterpret_cast<uint4*>(first ? fa : fb) + 2 * j;
      d[0] = lo;
      d[1] = hi;
    }
  }
}

// int8 -> bf16, exact (|q| <= 128 has at most 8 significant bits): the fp32
// value's upper 16 bits. n % 16 == 0, both pointers 16-byte aligned.
__global__ void __launch_bounds__(256) k_s8_to_bf16(const int8_t* __restrict__ q, __nv_bfloat16* __restrict__ w,
                                                    size_t n) {
  const size_t n16 = n / 16;
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n16; i += size_t(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(q) + i);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int b0 = int(int8_t(in[j] & 0xFFu)), b1 = int(int8_t((in[j] >> 8) & 0xFFu));
      const int b2 = int(int8_t((in[j] >> 16) & 0xFFu)), b3 = int(int8_t(in[j] >> 24));
      o[2 * j] = (__float_as_uint(float(b0)) >> 16) | (__float_as_uint(float(b1)) & 0xFFFF0000u);
      o[2 * j + 1] = (__float_as_uint(float(b2)) >> 16) | (__float_as_uint(float(b3)) & 0xFFFF0000u);
    }
    uint4* d = reinterpret_cast<uint4*>(w) + 2 * i;
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// 16-bit maps (f16 unless given), 128-byte swizzle, box of 64 elements (128 B)
// along K. 2-D: [rows][cols]; 3-D: [2][rows][cols] (gate half, up half).
bool sh_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t halves, uint32_t box_rows,
            CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  if (rows == 0) rows = 1;
  const cuuint64_t dims[3] = {cols, rows, halves};
  const cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  const cuuint32_t box[3] = {uint32_t(SKc), box_rows, uint32_t(halves)};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, halves > 1 ? 3 : 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool sh_supported(const v4moe_config& c, int64_t T) {
  return c.shared_inter > 0 && T >= kShMinTokens && c.shared_inter % 128 == 0 && c.hidden % 256 == 0 &&
         tensor_map_encoder() != nullptr;
}

size_t sh_extra_bytes(const v4moe_config& c, int64_t T) {
  if (c.shared_inter <= 0 || T < kShMinTokens) return 0;
  const size_t n13 = size_t(2) * c.shared_inter * c.hidden, n2 = size_t(c.hidden) * c.shared_inter;
  return align_up(n13 * 2) + align_up(n2 * 2);
}

namespace {

ShParams sh_params(const ForwardArgs& a, const int* sigma) {
  const v4moe_config& c = a.c;
  ShParams P = {};
  P.T = a.T;
  P.H = c.hidden;
  P.Is = c.shared_inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.limit = c.swiglu_limit;
  P.sigma = sigma;
  P.hs = reinterpret_cast<__half*>(a.hs);
  P.topk_ids = a.topk_ids;
  P.topk_w = a.topk_w;
  P.slot_pos = a.slot_pos;
  P.y_slot = a.y_slot;
  P.out = a.out;
  P.status = a.status;
  return P;
}

int sm_count() {
  const int sms = device_sms();
  return sms;
}

}  // namespace

cudaError_t launch_sh_w13(const ForwardArgs& a, const __half* x16, const int* sigma, char* extra, cudaStream_t st) {
  const v4moe_config& c = a.c;
  const int T = a.T, H = c.hidden, Is = c.shared_inter;
  const size_t n13 = size_t(2) * Is * H, n2 = size_t(H) * Is;
  __half* w13h = reinterpret_cast<__half*>(extra);
  __half* w2h = reinterpret_cast<__half*>(extra + align_up(n13 * 2));
  const int sms = sm_count();
  cudaError_t e = launch_kernel("sh_widen", k_s8_to_f16, dim3(4 * sms), dim3(256), 0, st, true, a.w.sh_w13, w13h, n13,
                                a.w.sh_w2, w2h, n2);
  if (e != cudaSuccess) return e;
  CUtensorMap mA, mB;
  if (!sh_map(&mA, x16, H, T, 1, SMt) || !sh_map(&mB, w13h, H, Is, 2, SNr / 2)) return cudaErrorInvalidValue;
  set_smem(k_sh_gemm, kSSmem);
  ShParams P = sh_params(a, sigma);
  P.mode = kSW13;
  P.nb = Is / (SNr / 2);
  P.ntiles = (T + SMt - 1) / SMt * P.nb;
  P.nk = H / SKc;
  P.scale = a.w.sh_w13_scale;
  return launch_kernel("sh_w13", k_sh_gemm, dim3(std::min(sms, P.ntiles)), dim3(kSThreads), kSSmem, st, true, P, mA,
                       mB);
}

cudaError_t launch_sh_w2_combine(const ForwardArgs& a, char* extra, cudaStream_t st) {
  const v4moe_config& c = a.c;
  const int T = a.T, H = c.hidden, Is = c.shared_inter;
  const __half* w2h = reinterpret_cast<const __half*>(extra + align_up(size_t(2) * Is * H * 2));
  CUtensorMap mA, mB;
  if (!sh_map(&mA, a.hs, Is, T, 1, SMt) || !sh_map(&mB, w2h, Is, H, 1, SNr)) return cudaErrorInvalidValue;
  set_smem(k_sh_gemm, kSSmem);
  ShParams P = sh_params(a, nullptr);
  P.mode = kSW2;
  P.nb = H / SNr;
  P.ntiles = (T + SMt - 1) / SMt * P.nb;
  P.nk = Is / SKc;
  P.scale = a.w.sh_w2_scale;
  return launch_kernel("sh_w2", k_sh_gemm, dim3(std::min(sm_count(), P.ntiles)), dim3(kSThreads), kSSmem, st, true,
                       P, mA, mB);
}

size_t linear_w8a16_ws_bytes(int64_t G, int64_t N, int64_t K) { return 256 + align_up(size_t(G) * N * K * 2); }

namespace {

// Weight rows per tile: 256 unless 128-row tiles fill the SMs' waves much
// better. A 128-row tile moves 4/3 the operand bytes per flop of a 256-row
// one and the GEMM is bound by that shared-memory fill rate: measured on B200
// (4096 x 1536 x 4096: 2 waves of 256-row tiles 0.060 ms, 3 waves of 128-row
// tiles 0.074 ms), a 128-row tile does ~0.6 of the work per unit time.
int lin_block_rows(int mt, int G, int N, int sms) {
  auto eff = [&](int bn) {
    const int nbg = (N + bn - 1) / bn;
    const double tiles = double(mt) * G * nbg;
    const double waves = std::ceil(tiles / sms);
    return tiles / (waves * sms) * double(N) / (double(nbg) * bn);
  };
  return eff(128) * 0.6 > eff(256) ? 128 : 256;
}

}  // namespace

cudaError_t launch_linear_w8a16(int T, int G, int N, int K, const __nv_bfloat16* x, const int8_t* q,
                                const float* scale, __nv_bfloat16* out, char* ws, cudaStream_t st) {
  __nv_bfloat16* qw = reinterpret_cast<__nv_bfloat16*>(ws + 256);
  const int sms = sm_count();
  cudaError_t e = launch_kernel("lin_widen", k_s8_to_bf16, dim3(4 * sms), dim3(256), 0, st, false, q, qw,
                                size_t(G) * N * K);
  if (e != cudaSuccess) return e;
  ShParams P = {};
  P.T = T;
  P.H = 0;
  P.G = G;
  P.N = N;
  P.K = K;
  P.mode = kSLin;
  P.mt = (T + SMt - 1) / SMt;
  P.bn = lin_block_rows(P.mt, G, N, sms);
  P.nbg = (N + P.bn - 1) / P.bn;
  P.nb = G * P.nbg;
  P.ntiles = P.mt * P.nb;
  // the operand with more bytes is read once: walk the token tiles of a weight
  // block first when the weights are the larger operand
  P.order = N > T ? 1 : 0;
  P.nk = K / SKc;
  P.scale = scale;
  P.out = out;
  P.status = reinterpret_cast<uint32_t*>(ws);
  CUtensorMap mA, mB;
  constexpr auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!sh_map(&mA, x, uint64_t(G) * K, T, 1, SMt, BF) || !sh_map(&mB, qw, K, uint64_t(G) * N, 1, P.bn, BF))
    return cudaErrorInvalidValue;
  set_smem(k_sh_gemm, kSSmem);
  return launch_kernel("lin_gemm", k_sh_gemm, dim3(std::min(sms, P.ntiles)), dim3(kSThreads), kSSmem, st, true, P,
                       mA, mB);
}

}  // namespace v4moe
