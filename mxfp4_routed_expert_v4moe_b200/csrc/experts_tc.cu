// Tensor-core expert path (more than 8 tokens): grouped GEMMs on tcgen05 with
// MXFP4 weights dequantised to f16 in shared memory and fp32 accumulation in
// tensor memory.
//
// What it computes ("Checked in its code" rows "SwiGLU feed-forward", "Shared
// expert"; "config.json" experts_w4a16 / linears_w8a16):
//   w13: per group (routed expert e, or the shared expert) and tile of 64
//        channels j and <= 128 tokens: [g; u] = W13[{j, I+j}] x_t (fp32),
//        h_t[j] = silu(min(g, L)) * clamp(u, -L, L), stored as f16;
//   w2:  per group and tile of 128 output rows m and <= 128 tokens:
//        y_t[m] = W2[m] h_t (fp32), stored per slot; a combine kernel then
//        forms out[t] = sum_j w[t,j] y_{slot(t,j)} + y_shared[t] in slot order.
//
// One persistent CTA per SM (384 threads, warp-specialised):
//   warp 0      TMA producer: activation tile (64 K x <= 128 rows, f16,
//               128-byte swizzle) and the weight-code tile of each K chunk;
//   warp 1      tcgen05.mma issuer (one thread) and TMEM owner;
//   warps 4-7   epilogue: tcgen05.ld of the fp32 accumulator, clamped SwiGLU
//               (w13) or the per-slot output rows (w2), global stores;
//   warps 8-11  dequantisers: one thread per weight row; E2M1 pairs -> exact
//               f16 (cvt.rn.f16x2.e2m1x2), E8M0 group scale applied as an
//               exact power of two relative to the row's largest group
//               exponent (the row factor 2^(Xmax-13) is applied by the
//               epilogue), int8 -> f16 exactly; written into shared memory in
//               the canonical K-major 128-byte-swizzled layout.
// Stages of A (dequantised weights), B (activations) and codes rotate through
// mbarriers; the fp32 accumulator (128 lanes x <= 128 columns) is double
// buffered in TMEM so the epilogue of one tile overlaps the next tile.
// Activations are f16 copies of the bf16 inputs scaled per token by a power of
// two (exact; the epilogue undoes it), h is f16.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int BM = 128;            // weight rows per tile
constexpr int BK = 64;             // K per stage (one 128-byte swizzle atom of f16)
constexpr int BN = 128;            // max tokens per tile
constexpr int kStages = 5;
constexpr int kThreads = 512;   // 16 warps: TMA, MMA, 2 idle, 4 epilogue, 8 dequantiser
constexpr uint32_t kTries = 1u << 21;

enum { kW13 = 0, kW2 = 1 };

// Shared memory layout (bytes, from a 1024-aligned base).
constexpr int kAStage = BM * BK * 2;      // 16 KB
constexpr int kBStage = BN * BK * 2;      // 16 KB
constexpr int kCStage = BM * 64;          // codes: 64 B per row (int8); fp4 uses 32
constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStages * kAStage;
constexpr int kOffC = kOffB + kStages * kBStage;
constexpr int kOffX = kOffC + kStages * kCStage;          // epilogue exchange [64][33] fp32
constexpr int kXchStride = 33;
constexpr int kOffInv = kOffX + 64 * kXchStride * 4;      // per-column token factors [2][BN]
constexpr int kOffBar = kOffInv + 2 * BN * 4;
constexpr int kSmemBytes = kOffBar + 256 + 1024;          // + barriers, + alignment slack

struct TcTile {
  int grp, row0, n0, n;
};

struct TcParams {
  int T, H, I, Is, E, k;
  float limit;
  int mode;
  int tail_tiles;                   // > 0: only the last tail_tiles tiles of the list (the shared expert's)
  const int32_t* offsets;
  const int32_t* sorted_slot;
  const int* sigma;                 // [T] token exponents of the f16 activations
  const TcTile* tiles;
  const int* ntiles;
  const uint8_t* w_codes;           // routed codes (w13 or w2), for L2 prefetch
  const uint8_t* sh_codes;          // shared int8 weights, for L2 prefetch
  const __half* b_routed;           // activations of routed groups (x in slot order, or h)
  const __half* b_shared;           // activations of the shared expert (x, or hs)
  const uint8_t* w_scales;          // routed E8M0 scales (w13 or w2)
  const float* sh_scale;            // shared expert fp32 row scales
  __half* h;                        // w13 out: [S, I]
  __half* hs;                       // w13 out: [T, Is]
  __nv_bfloat16* y_slot;            // w2 out: [S, H] bf16
  float* ys;                        // w2 out: [T, H]
  uint32_t* status;
};

struct TcBars {
  uint64_t full_b[kStages];
  uint64_t full_c[kStages];
  uint64_t full_a[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float pow2f(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((e + 127) << 23);
}

__device__ __forceinline__ bool wait_role(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  for (uint32_t i = 0; i < kTries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
  return false;
}

// Per-tile geometry shared by all roles.
struct TileGeo {
  bool shared;        // shared-expert group (int8 weights)
  int K;              // reduction length
  int nk;             // K chunks
  int brow0;          // first activation row of the tile (in the B tensor)
  int n, n_load, n_mma;
  int crow0, crow1;   // first code rows of the two 64-row halves
  int srow0, srow1;   // first scale rows (routed MX) of the halves
};

__device__ __forceinline__ TileGeo geo(const TcParams& P, const TcTile& t) {
  TileGeo g;
  g.shared = t.grp == P.E;
  g.n = t.n;
  g.n_load = (t.n + 31) / 32 * 32;
  g.n_mma = (t.n + 15) / 16 * 16;
  if (P.mode == kW13) {
    g.K = P.H;
    const int Ig = g.shared ? P.Is : P.I;
    const int base = g.shared ? 0 : t.grp * 2 * P.I;
    g.crow0 = base + t.row0;
    g.crow1 = base + Ig + t.row0;
  } else {
    g.K = g.shared ? P.Is : P.I;
    const int base = g.shared ? 0 : t.grp * P.H;
    g.crow0 = base + t.row0;
    g.crow1 = base + t.row0 + 64;
  }
  g.srow0 = g.crow0;
  g.srow1 = g.crow1;
  g.nk = g.K / BK;
  g.brow0 = (g.shared ? 0 : P.offsets[t.grp]) + t.n0;
  return g;
}

// Global weight row (for scales) of tile row r (0..127).
__device__ __forceinline__ int scale_row(const TileGeo& g, int r) { return r < 64 ? g.srow0 + r : g.srow1 + (r - 64); }

// Largest E8M0 exponent of a scale row of G bytes (G % 16 == 0 or small).
__device__ __forceinline__ int row_max_e8m0(const uint8_t* row, int G) {
  int m = 0;
  if ((G & 15) == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(row);
    uint32_t v = 0;
    for (int i = 0; i < G / 16; ++i) {
      const uint4 q = __ldg(p + i);
      v = __vmaxu4(v, __vmaxu4(__vmaxu4(q.x, q.y), __vmaxu4(q.z, q.w)));
    }
    m = max(max(int(v & 0xFF), int((v >> 8) & 0xFF)), max(int((v >> 16) & 0xFF), int(v >> 24)));
  } else {
    for (int i = 0; i < G; ++i) m = max(m, int(__ldg(row + i)));
  }
  return m;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_tc_gemm(TcParams P, const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
              const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcBars& B = *reinterpret_cast<TcBars*>(smem + kOffBar);
  volatile int* abort_flag = &B.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&B.full_b[s], 1);
      mbar_init(&B.full_c[s], 1);
      mbar_init(&B.full_a[s], 8);  // one arrival per dequantiser warp
      mbar_init(&B.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.acc_full[b], 1);
      mbar_init(&B.acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&B.done, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&B.tmem_base, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;
  pdl_wait();  // tiles, routing and activations come from earlier kernels
  const int ntiles = *P.ntiles;
  const int tile0 = P.tail_tiles > 0 ? max(0, ntiles - P.tail_tiles) : 0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_tmap(&tmB_r);
    prefetch_tmap(&tmB_s);
    prefetch_tmap(&tmC_r);
    prefetch_tmap(&tmC_s);
    uint32_t gc = 0;  // global chunk counter
    bool ok = true;
    for (int ti = tile0 + int(blockIdx.x); ti < ntiles && ok; ti += gridDim.x) {
      const TcTile t = P.tiles[ti];
      const TileGeo g = geo(P, t);
      const void* tmB = g.shared ? static_cast<const void*>(&tmB_s) : static_cast<const void*>(&tmB_r);
      const void* tmC = g.shared ? static_cast<const void*>(&tmC_s) : static_cast<const void*>(&tmC_r);
      const int cb = g.shared ? 64 : 32;  // code bytes per row per chunk
      // Move the next tile's weights (and its activations, when they change)
      // towards L2 now, so that its TMA loads do not wait on DRAM.
      const int tn = ti + int(gridDim.x);
      if (tn < ntiles) {
        const TcTile t2 = P.tiles[tn];
        const TileGeo g2 = geo(P, t2);
        const size_t rb = g2.shared ? size_t(g2.K) : size_t(g2.K / 2);
        const uint8_t* wb = g2.shared ? P.sh_codes : P.w_codes;
        prefetch_l2_range(wb + size_t(g2.crow0) * rb, 64 * rb);
        prefetch_l2_range(wb + size_t(g2.crow1) * rb, 64 * rb);
        if (!g2.shared) {
          const size_t G = size_t(g2.K / 32);
          prefetch_l2_range(P.w_scales + size_t(g2.srow0) * G, 64 * G);
          prefetch_l2_range(P.w_scales + size_t(g2.srow1) * G, 64 * G);
        }
        if (t2.grp != t.grp || t2.n0 != t.n0) {
          const __half* bb = g2.shared ? P.b_shared : P.b_routed;
          prefetch_l2_range(bb + size_t(g2.brow0) * g2.K, size_t(t2.n) * g2.K * 2);
        }
      }
      for (int c = 0; c < g.nk; ++c, ++gc) {
        const int s = gc % kStages;
        const uint32_t u = gc / kStages;
        if (!wait_role(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        char* bs = smem + kOffB + s * kBStage;
        mbar_arrive_expect_tx(&B.full_b[s], uint32_t(g.n_load * BK * 2));
        for (int i = 0; i < g.n_load / 32; ++i) tma_load_2d(bs + i * 4096, tmB, c * BK, g.brow0 + 32 * i, &B.full_b[s]);
        char* cs = smem + kOffC + s * kCStage;
        mbar_arrive_expect_tx(&B.full_c[s], uint32_t(BM * cb));
        tma_load_2d(cs, tmC, c * cb, g.crow0, &B.full_c[s]);
        tma_load_2d(cs + 64 * cb, tmC, c * cb, g.crow1, &B.full_c[s]);
      }
    }
    // copies still in flight land before the CTA leaves (only after an abort
    // can a stage be armed and not consumed)
    for (uint32_t q = 0; q < uint32_t(kStages) && q < gc; ++q) {
      const uint32_t gq = gc - 1 - q;
      mbar_wait_bounded(&B.full_b[gq % kStages], (gq / kStages) & 1u, kTries);
      mbar_wait_bounded(&B.full_c[gq % kStages], (gq / kStages) & 1u, kTries);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t gc = 0, lt = 0;
    bool ok = true;
    for (int ti = tile0 + int(blockIdx.x); ti < ntiles && ok; ti += gridDim.x, ++lt) {
      const TcTile t = P.tiles[ti];
      const TileGeo g = geo(P, t);
      const uint32_t b = lt & 1u, v = lt >> 1;
      if (!wait_role(&B.acc_empty[b], (v & 1u) ^ 1u, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t d = tmem + b * BN;
      const uint32_t idesc = idesc_f16_f32(BM, g.n_mma);
      for (int c = 0; c < g.nk; ++c, ++gc) {
        const int s = gc % kStages;
        const uint32_t u = gc / kStages;
        if (!wait_role(&B.full_a[s], u & 1u, abort_flag, P.status) ||
            !wait_role(&B.full_b[s], u & 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + kOffA + s * kAStage);
        const uint32_t b0 = smem_u32(smem + kOffB + s * kBStage);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_f16_ss(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                      (c > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&B.empty[s]);
      }
      if (!ok) break;
      umma_commit(&B.acc_full[b]);
    }
    // all MMAs issued by this thread are complete before TMEM is released
    umma_commit(&B.done);
    mbar_wait_bounded(&B.done, 0, kTries);
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dequantisers
    const int dq = threadIdx.x - 256;
    const int r = dq >> 1;   // tile row
    const int hf = dq & 1;   // half of the 64-element chunk: elements [32 hf, 32 hf + 32)
    uint32_t gc = 0;
    bool ok = true;
    for (int ti = tile0 + int(blockIdx.x); ti < ntiles && ok; ti += gridDim.x) {
      const TcTile t = P.tiles[ti];
      const TileGeo g = geo(P, t);
      int xmax = 0;
      const uint8_t* srow = nullptr;
      const int G = g.K / 32;
      const bool vec = (G & 15) == 0;  // scale rows read 16 bytes (8 chunks) at a time
      uint4 win = make_uint4(0, 0, 0, 0), nxt = win;
      if (!g.shared) {
        srow = P.w_scales + size_t(scale_row(g, r)) * G;
        if (vec) {
          win = __ldg(reinterpret_cast<const uint4*>(srow));
          if (G > 16) nxt = __ldg(reinterpret_cast<const uint4*>(srow) + 1);
        }
        xmax = row_max_e8m0(srow, G);
      }
      for (int c = 0; c < g.nk; ++c, ++gc) {
        if (!g.shared && vec && c > 0 && (c & 7) == 0) {
          win = nxt;
          if ((c / 8 + 1) * 16 < G) nxt = __ldg(reinterpret_cast<const uint4*>(srow) + c / 8 + 1);
        }
        const int s = gc % kStages;
        const uint32_t u = gc / kStages;
        if (!wait_role(&B.full_c[s], u & 1u, abort_flag, P.status) ||
            !wait_role(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        const char* cs = smem + kOffC + s * kCStage;
        uint32_t w[16];
        if (!g.shared) {
          const uint4 q = *reinterpret_cast<const uint4*>(cs + r * 32 + hf * 16);
          uint32_t e8;  // scale byte of group 2c + hf
          if (vec) {
            const uint32_t wv = (c & 4) ? ((c & 2) ? win.w : win.z) : ((c & 2) ? win.y : win.x);
            e8 = (wv >> ((c & 1) * 16 + hf * 8)) & 0xFFu;
          } else {
            e8 = __ldg(srow + 2 * c + hf);
          }
          const uint32_t sc = f16_pow2_bits(int(e8) - xmax + 13) * 0x10001u;
          const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t f[4];
            e2m1x8_to_f16x2(qq[i], f);
#pragma unroll
            for (int j = 0; j < 4; ++j) w[4 * i + j] = hmul2_u32(f[j], sc);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint4 q = *reinterpret_cast<const uint4*>(cs + r * 64 + hf * 32 + 16 * i);
            s8x4_to_f16x2(q.x, w[8 * i + 0], w[8 * i + 1]);
            s8x4_to_f16x2(q.y, w[8 * i + 2], w[8 * i + 3]);
            s8x4_to_f16x2(q.z, w[8 * i + 4], w[8 * i + 5]);
            s8x4_to_f16x2(q.w, w[8 * i + 6], w[8 * i + 7]);
          }
        }
        char* as = smem + kOffA + s * kAStage + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ch = 4 * hf + j;  // 16-byte chunk within the row
          *reinterpret_cast<uint4*>(as + ((ch ^ (r & 7)) << 4)) =
              make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
        fence_proxy_async_smem();  // make this thread's generic-proxy writes visible to the MMA
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.full_a[s]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;          // TMEM lane quarter
    const int er = threadIdx.x - 128;  // 0..127
    float* xch = reinterpret_cast<float*>(smem + kOffX);
    float* inv = reinterpret_cast<float*>(smem + kOffInv);
    uint32_t lt = 0;
    for (int ti = tile0 + int(blockIdx.x); ti < ntiles; ti += gridDim.x, ++lt) {
      const TcTile t = P.tiles[ti];
      const TileGeo g = geo(P, t);
      const uint32_t b = lt & 1u, v = lt >> 1;
      const int row = 32 * q + lane;  // tile row of this thread
      // row factor (weights) of this thread's row
      float rowf;
      if (!g.shared) {
        const int G = g.K / 32;
        rowf = pow2f(row_max_e8m0(P.w_scales + size_t(scale_row(g, row)) * G, G) - 127 - 13);
      } else {
        rowf = __ldg(P.sh_scale + (row < 64 ? g.crow0 + row : g.crow1 + row - 64));
      }
      // per-column token factor (w13: undo the activation scaling)
      float* inv_b = inv + b * BN;
      if (P.mode == kW13) {
        float f = 1.0f;
        if (er < g.n) {
          const int tok = g.shared ? t.n0 + er : P.sorted_slot[g.brow0 + er] / P.k;
          f = pow2f(-P.sigma[tok]);
        }
        inv_b[er] = f;
      }
      const bool got = wait_role(&B.acc_full[b], v & 1u, abort_flag, P.status);
      named_bar_sync(1, 128);
      if (!got || *abort_flag) break;
      tc_fence_after();
      const uint32_t acc = tmem + b * BN + (uint32_t(32 * q) << 16);
      for (int c0 = 0; c0 < g.n; c0 += 32) {
        uint32_t rv[32];
        tmem_ld_32x32b_x32(acc + c0, rv);
        tmem_wait_ld();
        if (P.mode == kW13) {
          if (q >= 2) {
#pragma unroll
            for (int i = 0; i < 32; ++i) xch[((q - 2) * 32 + lane) * kXchStride + i] = __uint_as_float(rv[i]) * rowf;
          }
          named_bar_sync(1, 128);
          if (q < 2) {
            const int Ig = g.shared ? P.Is : P.I;
            __half* hout = g.shared ? P.hs : P.h;
            const int ch = t.row0 + 32 * q + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = c0 + i;
              if (col < g.n) {
                const float f = inv_b[col];
                const float gv = __uint_as_float(rv[i]) * rowf * f;
                const float uv = xch[(q * 32 + lane) * kXchStride + i] * f;
                hout[size_t(g.brow0 + col) * Ig + ch] = __float2half_rn(clamped_swiglu_f(gv, uv, P.limit));
              }
            }
          }
          named_bar_sync(1, 128);
        } else {
          const int m = t.row0 + row;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = c0 + i;
            if (col < g.n) {
              const float v = __uint_as_float(rv[i]) * rowf;
              if (g.shared)
                P.ys[size_t(g.brow0 + col) * P.H + m] = v;
              else
                P.y_slot[size_t(g.brow0 + col) * P.H + m] = __float2bfloat16_rn(v);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// ------------------------------------------------------------------ helpers

// x -> f16 (per-token power-of-two scale) in natural K order: x16[t] and its
// copies in sorted-slot order xperm[slot_pos[t*k+j]]. One warp per token.
__global__ void __launch_bounds__(256) k_tc_gather(int T, int H, int E, int k, const __nv_bfloat16* __restrict__ x,
                                                   const int32_t* __restrict__ topk_ids,
                                                   const int32_t* __restrict__ slot_pos, __half* __restrict__ x16,
                                                   __half* __restrict__ xperm, int* __restrict__ sigma) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const uint4* s4 = reinterpret_cast<const uint4*>(x + size_t(t) * H);
  uint32_t mx = 0;
#pragma unroll 4
  for (int p = lane; p < H / 8; p += 32) {
    const uint4 v = __ldg(s4 + p);
    mx = max(mx, max(max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu), max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu)));
    mx = max(mx, max(max(v.z & 0x7FFFu, (v.z >> 16) & 0x7FFFu), max(v.w & 0x7FFFu, (v.w >> 16) & 0x7FFFu)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int ef = int(mx >> 7);
  int sg = 0;
  if (mx != 0) sg = ef == 0 ? 120 : 141 - ef;
  sg = max(-120, min(120, sg));
  if (lane == 0) sigma[t] = sg;
  const float mul = __int_as_float((sg + 127) << 23);
  int dst[8];
  int nd = 0;
  for (int j = 0; j < k; ++j) {
    const int e = topk_ids[size_t(t) * k + j];
    if (e >= 0 && e < E) dst[nd++] = slot_pos[size_t(t) * k + j];
  }
#pragma unroll 2
  for (int p = lane; p < H / 8; p += 32) {
    const uint4 v = __ldg(s4 + p);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hv = __floats2half2_rn(__uint_as_float(in[i] << 16) * mul, __uint_as_float(in[i] & 0xFFFF0000u) * mul);
      ow[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    reinterpret_cast<uint4*>(x16 + size_t(t) * H)[p] = o;
    for (int j = 0; j < nd; ++j) reinterpret_cast<uint4*>(xperm + size_t(dst[j]) * H)[p] = o;
  }
}

// Tile lists of both GEMMs (one CTA): per group (routed experts in id order,
// then the shared expert unless Is == 0), token tiles of <= BN, times the row
// blocks: for the routed experts rb13 channels (w13) and rb2 output rows (w2),
// for the shared expert 64 channels and 128 rows. One thread counts a group's
// tiles, the counts are prefix-summed across the block, and one warp writes a
// group's entries.
__device__ __forceinline__ int block_excl_scan_1024(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_tot[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  return warp_tot[warp] + incl - v;
}

__global__ void __launch_bounds__(1024) k_tc_tiles(int T, int E, int H, int I, int Is, int rb13, int rb2, int tn,
                                                   const int32_t* __restrict__ offsets,
                                                   TcTile* __restrict__ t13, int* __restrict__ n13, TcTile* __restrict__ t2,
                                                   int* __restrict__ n2) {
  __shared__ int wt13[32], wt2[32];
  __shared__ int tot13, tot2;
  __shared__ int gn[1025], gb13[1025], gb2[1025];
  const int G = E + (Is > 0 ? 1 : 0);  // <= 1025 groups: threads take g and g + 1024
  int c13[2] = {0, 0}, c2[2] = {0, 0};
  for (int q = 0; q < 2; ++q) {
    const int g = threadIdx.x + q * 1024;
    if (g < G) {
      const int n = g < E ? offsets[g + 1] - offsets[g] : T;
      const int tile = g < E ? tn : BN;
      const int tt = (n + tile - 1) / tile;
      gn[g] = n;
      c13[q] = tt * (g < E ? I / rb13 : Is / 64);
      c2[q] = tt * (g < E ? H / rb2 : H / 128);
    }
  }
  // the second group of a thread (only the shared expert when E == 1024) follows all first groups
  const int b13 = block_excl_scan_1024(c13[0], wt13, &tot13);
  const int b2 = block_excl_scan_1024(c2[0], wt2, &tot2);
  if (threadIdx.x < G) {
    gb13[threadIdx.x] = b13;
    gb2[threadIdx.x] = b2;
  }
  if (threadIdx.x == 0) {
    if (G > 1024) {
      gb13[1024] = tot13;
      gb2[1024] = tot2;
    }
    *n13 = tot13 + c13[1];
    *n2 = tot2 + c2[1];
  }
  __syncthreads();
  // one warp per group, its lanes over the group's tiles (token tile major,
  // then row block)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int g = warp; g < G; g += 32) {
    const int n = gn[g];
    const int tile = g < E ? tn : BN;
    const int tt = (n + tile - 1) / tile;
    const int r13 = g < E ? rb13 : 64, r2 = g < E ? rb2 : 128;
    const int nb13 = (g < E ? I : Is) / r13, nb2 = H / r2;
    for (int i = lane; i < tt * nb13; i += 32) {
      const int n0 = (i / nb13) * tile;
      t13[gb13[g] + i] = TcTile{g, (i % nb13) * r13, n0, min(tile, n - n0)};
    }
    for (int i = lane; i < tt * nb2; i += 32) {
      const int n0 = (i / nb2) * tile;
      t2[gb2[g] + i] = TcTile{g, (i % nb2) * r2, n0, min(tile, n - n0)};
    }
  }
}

// ------------------------------------------------------------------ host

// 2-D map over a row-major [rows, cols] tensor; box {box_cols, box_rows}.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  if (rows == 0) rows = 1;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * uint64_t(esize)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Token tiles of the lists: at most S / kMxSmallTile + E routed ones (each
// expert's partial tile) plus the shared expert's T / BN (+ 1).
static int64_t tile_rows(const v4moe_config& c, int64_t T) {
  const int64_t S = T * c.top_k;
  return (S + kMxSmallTile - 1) / kMxSmallTile + c.n_experts + (T + BN - 1) / BN + 2;
}

size_t tc_extra_bytes(const v4moe_config& c, int64_t T) {
  const int64_t S = T * c.top_k;
  const int64_t tiles13 = tile_rows(c, T) * (std::max(c.inter, c.shared_inter) / 64);
  const int64_t tiles2 = tile_rows(c, T) * (c.hidden / 128);
  return align_up(size_t(S) * c.hidden * 2) + align_up(size_t(tiles13) * sizeof(TcTile)) +
         align_up(size_t(tiles2) * sizeof(TcTile)) + 256 + 2 * align_up(size_t(S) * (c.hidden / 32)) +
         2 * align_up(size_t(S) * (c.inter / 32));
}

cudaError_t launch_forward_tc(const ForwardArgs& a, __half* x16, int* sigma, char* extra, char* sh16,
                              cudaStream_t st) {
  const v4moe_config& c = a.c;
  const int T = a.T;
  const int64_t S = int64_t(T) * c.top_k;
  __half* xperm = reinterpret_cast<__half*>(extra);
  char* p = extra + align_up(size_t(S) * c.hidden * 2);
  const int64_t tiles13 = tile_rows(c, T) * (std::max(c.inter, c.shared_inter) / 64);
  TcTile* t13 = reinterpret_cast<TcTile*>(p);
  p += align_up(size_t(tiles13) * sizeof(TcTile));
  const int64_t tiles2 = tile_rows(c, T) * (c.hidden / 128);
  TcTile* t2 = reinterpret_cast<TcTile*>(p);
  p += align_up(size_t(tiles2) * sizeof(TcTile));
  int* counts = reinterpret_cast<int*>(p);  // [0] = n13, [1] = n2
  p += 256;
  // Routed experts on block-scaled MMA when the weights allow it: the
  // activation planes take the place of the f16 slot copies, the intermediate
  // planes that of the f16 intermediates.
  const bool mx = mx_supported(c, a.w);
  MxBuffers mb;
  mb.xq_hi = reinterpret_cast<uint8_t*>(xperm);
  mb.xq_lo = mb.xq_hi + size_t(S) * c.hidden;
  mb.hq_hi = reinterpret_cast<uint8_t*>(a.h);
  mb.hq_lo = mb.hq_hi + size_t(S) * c.inter;
  mb.xs_hi = reinterpret_cast<uint8_t*>(p);
  p += align_up(size_t(S) * (c.hidden / 32));
  mb.xs_lo = reinterpret_cast<uint8_t*>(p);
  p += align_up(size_t(S) * (c.hidden / 32));
  mb.hs_hi = reinterpret_cast<uint8_t*>(p);
  p += align_up(size_t(S) * (c.inter / 32));
  mb.hs_lo = reinterpret_cast<uint8_t*>(p);
  // Shared expert on its own f16 GEMM (large batches, block-scaled path only);
  // otherwise its tiles trail the routed ones in the lists.
  const bool shx = mx && sh_supported(c, T);
  const int tt_sh = c.shared_inter > 0 && !shx ? (T + BN - 1) / BN : 0;
  const int sh13 = tt_sh * (c.shared_inter / 64), sh2 = tt_sh * (c.hidden / 128);

  cudaError_t e = mx ? launch_mx_gather(a, x16, sigma, mb, st)
                     : launch_kernel("tc_gather", k_tc_gather, dim3((T + 7) / 8), dim3(256), 0, st, false, T,
                                     c.hidden, c.n_experts, c.top_k, a.x, a.topk_ids, a.slot_pos, x16, xperm, sigma);
  if (e != cudaSuccess) return e;
  // Token-major block-scaled tiles (128 slots x 256 weight rows) once the
  // experts average enough tokens to fill them; weight-major ones otherwise.
  const bool mxt = mx && int64_t(T) * c.top_k >= int64_t(kMxtMinAvg) * c.n_experts;
  // token tile of the routed groups: small for weight-major tiles of few tokens
  const int tn = mx && !mxt && int64_t(T) * c.top_k < int64_t(kMxSmallAvg) * c.n_experts ? kMxSmallTile : BN;
  e = launch_kernel("tc_tiles", k_tc_tiles, dim3(1), dim3(1024), 0, st, false, T, c.n_experts, c.hidden, c.inter,
                    shx ? 0 : c.shared_inter, mxt ? 128 : 64, mxt ? 256 : 128, tn, a.offsets, t13, counts, t2,
                    counts + 1);
  if (e != cudaSuccess) return e;

  // tensor maps
  const int Isx = c.shared_inter > 0 ? c.shared_inter : 64;
  CUtensorMap mB_r13, mB_s13, mC_r13, mC_s13, mB_r2, mB_s2, mC_r2, mC_s2;
  bool ok = true;
  ok &= make_map(&mB_r13, xperm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c.hidden, S, BK, 32,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mB_s13, x16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c.hidden, T, BK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mC_r13, a.w.w13_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, c.hidden / 2,
                 uint64_t(c.n_experts) * 2 * c.inter, 32, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
  ok &= make_map(&mB_r2, a.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c.inter, S, BK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mC_r2, a.w.w2_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, c.inter / 2,
                 uint64_t(c.n_experts) * c.hidden, 32, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (c.shared_inter > 0) {
    ok &= make_map(&mC_s13, a.w.sh_w13, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, c.hidden, 2 * uint64_t(c.shared_inter), 64,
                   64, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= make_map(&mB_s2, a.hs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, c.shared_inter, T, BK, 32,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&mC_s2, a.w.sh_w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, c.shared_inter, c.hidden, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    mC_s13 = mC_r13;
    mB_s2 = mB_r2;
    mC_s2 = mC_r2;
  }
  (void)Isx;
  if (!ok) return cudaErrorInvalidValue;

  const int sms = device_sms();
  set_smem(k_tc_gemm, kSmemBytes);

  TcParams P;
  P.T = T;
  P.H = c.hidden;
  P.I = c.inter;
  P.Is = c.shared_inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.limit = c.swiglu_limit;
  P.offsets = a.offsets;
  P.sorted_slot = a.sorted_slot;
  P.sigma = sigma;
  P.status = a.status;
  P.h = reinterpret_cast<__half*>(a.h);
  P.hs = reinterpret_cast<__half*>(a.hs);
  P.y_slot = a.y_slot;
  P.ys = a.ys;

  P.tail_tiles = 0;
  P.mode = kW13;
  P.w_codes = a.w.w13_codes;
  P.sh_codes = reinterpret_cast<const uint8_t*>(a.w.sh_w13);
  P.b_routed = xperm;
  P.b_shared = x16;
  P.tiles = t13;
  P.ntiles = counts;
  P.w_scales = a.w.w13_scales;
  P.sh_scale = a.w.sh_w13_scale;
  if (mx) {
    e = mxt ? launch_mxt_gemm(a, 0, t13, counts, sh13, mb, st)
            : launch_mx_gemm(a, 0, t13, counts, sh13, tn, mb, st);
    if (e != cudaSuccess) return e;
    P.tail_tiles = sh13;
    if (shx && (e = launch_sh_w13(a, x16, sigma, sh16, st)) != cudaSuccess) return e;
  }
  if (!mx || sh13 > 0) {
    e = launch_kernel("tc_w13", k_tc_gemm, dim3(sms), dim3(kThreads), kSmemBytes, st, true, P, mB_r13, mB_s13,
                      mC_r13, mC_s13);
    if (e != cudaSuccess) return e;
  }

  P.mode = kW2;
  P.w_codes = a.w.w2_codes;
  P.sh_codes = reinterpret_cast<const uint8_t*>(a.w.sh_w2);
  P.b_routed = reinterpret_cast<const __half*>(a.h);
  P.b_shared = reinterpret_cast<const __half*>(a.hs);
  P.tiles = t2;
  P.ntiles = counts + 1;
  P.w_scales = a.w.w2_scales;
  P.sh_scale = a.w.sh_w2_scale;
  if (mx) {
    e = mxt ? launch_mxt_gemm(a, 1, t2, counts + 1, sh2, mb, st)
            : launch_mx_gemm(a, 1, t2, counts + 1, sh2, tn, mb, st);
    if (e != cudaSuccess) return e;
    P.tail_tiles = sh2;
    if (shx) return launch_sh_w2_combine(a, sh16, st);  // the combine is in its epilogue
  }
  if (!mx || sh2 > 0) {
    e = launch_kernel("tc_w2", k_tc_gemm, dim3(sms), dim3(kThreads), kSmemBytes, st, true, P, mB_r2, mB_s2, mC_r2,
                      mC_s2);
    if (e != cudaSuccess) return e;
  }
  return launch_combine(a, st);
}

}  // namespace v4moe
