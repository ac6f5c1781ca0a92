// Routed experts on block-scaled tensor cores: tcgen05.mma kind::mxf8f6f4
// with the MXFP4 weights as the A operand exactly as stored (E2M1 codes,
// E8M0 scale per 32 K) and the activations as the B operand, split exactly
// into two E4M3 planes with E8M0 scales per 32 K.
//
// What it computes ("Checked in its code" row "SwiGLU feed-forward";
// "config.json" experts_w4a16): for every routed expert e and its tokens
// (slots in expert order),
//   w13: [g; u] = W13_e[{j, I+j}] x (fp32), h = silu(min(g, L)) * clamp(u, -L, L);
//   w2:  y_slot = bf16(W2_e h); the combine forms the output.
//
// Exact activations: a bf16 value has 8 significant bits. Per block of 32
// values with largest magnitude a, the scale 2^s (s the smallest exponent with
// a <= 448 * 2^s) takes the block into E4M3 range; hi = RN_e4m3(x / 2^s) keeps
// the top 4 bits and the residual x - hi 2^s (at most 4 bits, magnitude below
// 16 * 2^s) is lo * 2^(s-4) exactly, so x = hi 2^s + lo 2^(s-4) for every value
// within 2^-14 of the block maximum (smaller ones keep at least their top
// bits). Each K step is two MMAs, one per plane, accumulating in fp32 in TMEM.
// The intermediates h are split the same way by the w13 epilogue.
//
// One persistent CTA per SM (384 threads, warp-specialised):
//   warp 0      TMA producer: per 128-wide K chunk, the weight rows (E2M1
//               codes through a 16U4_ALIGN16B tensor map, expanded to 16-byte
//               groups, 128-byte swizzle) and both activation planes;
//   warp 1      TMEM owner and tcgen05.mma issuer (one thread);
//   warps 4-7   epilogue (TMEM lane quarters): clamped SwiGLU and the h planes
//               (w13) or the per-slot output rows (w2);
//   warps 8-11  scale writers: per chunk, the E8M0 scales of the 128 weight rows
//               and of the tile's tokens (both planes) into TMEM with
//               tcgen05.st, in the layout the block-scaled MMA reads (row
//               32 i + l of the operand in lane l of every lane quarter,
//               column i; one byte per K step of 32).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "launch.cuh"
#include "ptx.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int MBM = 128;       // weight rows per tile
constexpr int MBK = 128;       // K per stage (4 MMA steps of 32)
constexpr int MBN = 128;       // max tokens per tile
constexpr int kMMaxStages = 12;
constexpr int kMThreads = 384;
constexpr uint32_t kMTries = 1u << 21;

enum { kMW13 = 0, kMW2 = 1 };

// Shared memory: nst stages of [A: 128 weight rows x 128 K, E2M1 codes
// expanded to one byte each (16 KB)][activation hi plane: bn rows x 128 B]
// [lo plane], then the epilogue exchange and the barriers. bn (the token
// tile, a multiple of 32 up to MBN) and nst are chosen per launch: small
// token tiles leave room for a deeper ring.
constexpr int kMA = MBM * MBK;
constexpr int kMXch = 33;
constexpr int kMXchBytes = 128 * kMXch * 4;  // epilogue exchange [128][33] fp32
constexpr int kMSmemMax = 232448;           // dynamic shared memory per block
__host__ __device__ constexpr int mx_stage_bytes(int bn) { return kMA + 2 * bn * MBK; }
// Scale slot (two of them, each covering four K chunks): 16 bytes per weight
// row, then per token of the hi and the lo plane, brought in by TMA.
__host__ __device__ constexpr int mx_scale_slot(int bn) { return 16 * (MBM + 2 * bn); }

// TMEM columns: two accumulators of MBN, then 12 scale columns per stage.
constexpr uint32_t kMColSF = 2 * MBN;
constexpr uint32_t kMTmemCols = 512;
static_assert(kMColSF + 12 * kMMaxStages <= kMTmemCols, "TMEM columns");

struct MxTile {
  int grp, row0, n0, n;
};

struct MxParams {
  int T, H, I, E, k;
  float limit;
  int mode;
  int bn;   // token tile (rows of an activation plane per stage)
  int nst;  // ring stages
  const int32_t* offsets;
  const MxTile* tiles;
  const int* ntiles;      // tile count of the list (routed tiles come first)
  int shared_tiles;       // trailing tiles of the list that belong to the shared expert
  const uint8_t* w_scales;  // E8M0 [rows][K/32] of the routed weights (w13 or w2)
  const uint8_t* b_sc_hi;   // activation scales [slots][K/32] (x or h)
  const uint8_t* b_sc_lo;
  uint8_t* h_hi;            // w13 out: [S, I] E4M3
  uint8_t* h_lo;
  uint8_t* hs_hi;           // w13 out: [S, I/32] E8M0
  uint8_t* hs_lo;
  __nv_bfloat16* y_slot;    // w2 out: [S, H] bf16
  uint32_t* status;
};

struct MxBars {
  uint64_t full[kMMaxStages];
  uint64_t sf_full[kMMaxStages];
  uint64_t empty[kMMaxStages];
  uint64_t sc_full[2];
  uint64_t sc_empty[2];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

constexpr int kMBarBytes = (int(sizeof(MxBars)) + 127) / 128 * 128;

// This CTA's tiles (list positions blockIdx.x + i * gridDim.x) with their first
// activation row, copied into shared memory before the first TMA copy: every
// role walks them, and on this GPU a global load waits behind the SM's copies
// in flight. Past kTileCache tiles the list is read from global memory.
constexpr int kTileCache = 256;
struct TileCache {
  MxTile t[kTileCache];
  int brow0[kTileCache];
};
constexpr int kTileCacheBytes = int(sizeof(TileCache));

// Whole CTA; returns the number of this CTA's tiles.
__device__ __forceinline__ int cache_tiles(const MxParams& P, int ntiles, TileCache& C) {
  const int nmine = int(blockIdx.x) < ntiles ? (ntiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  for (int i = threadIdx.x; i < nmine && i < kTileCache; i += blockDim.x) {
    const MxTile t = P.tiles[blockIdx.x + i * gridDim.x];
    C.t[i] = t;
    C.brow0[i] = P.offsets[t.grp] + t.n0;
  }
  __syncthreads();
  return nmine;
}

__device__ __forceinline__ MxTile tile_at(const MxParams& P, const TileCache& C, int i, int& brow0) {
  if (i < kTileCache) {
    brow0 = C.brow0[i];
    return C.t[i];
  }
  const MxTile t = P.tiles[blockIdx.x + i * gridDim.x];
  brow0 = P.offsets[t.grp] + t.n0;
  return t;
}

__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  for (uint32_t i = 0; i < kMTries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
  return false;
}

// ------------------------------------------------------------------ E4M3 planes

__device__ __forceinline__ float exp2i(int s) { return __int_as_float((max(-126, min(127, s)) + 127) << 23); }

// Block exponent s (as E8M0 byte s + 127) for a block whose largest magnitude
// has float bits `amax_bits`: the smallest s with amax <= 448 * 2^s.
__device__ __forceinline__ int block_exp(uint32_t amax_bits) {
  if (amax_bits == 0) return 0;
  const float a = __uint_as_float(amax_bits);
  const int ea = int((amax_bits >> 23) & 0xFF) - 127;  // floor(log2 a) for normal a
  int s = ea - 8;
  if (a > 448.0f * exp2i(max(-126, min(126, s)))) ++s;
  return max(-126, min(122, s));
}

// Splits x (fp32, exactly a bf16 or f16 value) into E4M3 bytes hi, lo with
// x = hi 2^s + lo 2^(s-4).
__device__ __forceinline__ void split_e4m3(float x, int s, uint8_t& hi, uint8_t& lo) {
  const __nv_fp8_storage_t h = __nv_cvt_float_to_fp8(x * exp2i(-s), __NV_SATFINITE, __NV_E4M3);
  const __half_raw hr = __nv_cvt_fp8_to_halfraw(h, __NV_E4M3);
  const float r = x - __half2float(__half(hr)) * exp2i(s);
  hi = h;
  lo = __nv_cvt_float_to_fp8(r * exp2i(4 - s), __NV_SATFINITE, __NV_E4M3);
}

// x rows -> both planes and their scales, in slot order (copy t of a token
// goes to slot_pos[t k + j]); also the f16 copy x16 with a per-token power of
// two (sigma) for the shared expert's tiles. One warp per token.
__global__ void __launch_bounds__(256) k_mx_gather(int T, int H, int E, int k, const __nv_bfloat16* __restrict__ x,
                                                   const int32_t* __restrict__ topk_ids,
                                                   const int32_t* __restrict__ slot_pos, __half* __restrict__ x16,
                                                   int* __restrict__ sigma, uint8_t* __restrict__ xq_hi,
                                                   uint8_t* __restrict__ xq_lo, uint8_t* __restrict__ xs_hi,
                                                   uint8_t* __restrict__ xs_lo) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const uint4* s4 = reinterpret_cast<const uint4*>(x + size_t(t) * H);
  uint32_t mx = 0;
  for (int p = lane; p < H / 8; p += 32) {
    const uint4 v = __ldg(s4 + p);
    mx = max(mx, max(max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu), max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu)));
    mx = max(mx, max(max(v.z & 0x7FFFu, (v.z >> 16) & 0x7FFFu), max(v.w & 0x7FFFu, (v.w >> 16) & 0x7FFFu)));
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  const int ef = int(mx >> 7);
  int sg = 0;
  if (mx != 0) sg = ef == 0 ? 120 : 141 - ef;
  sg = max(-120, min(120, sg));
  if (lane == 0) sigma[t] = sg;
  const float mul = exp2i(sg);
  int dst[8];
  int nd = 0;
  for (int j = 0; j < k; ++j) {
    const int e = topk_ids[size_t(t) * k + j];
    if (e >= 0 && e < E) dst[nd++] = slot_pos[size_t(t) * k + j];
  }
  for (int p = lane; p < H / 8; p += 32) {
    const uint4 v = __ldg(s4 + p);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(in[i] << 16);
      f[2 * i + 1] = __uint_as_float(in[i] & 0xFFFF0000u);
    }
    // f16 copy for the shared expert
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hv = __floats2half2_rn(f[2 * i] * mul, f[2 * i + 1] * mul);
      ow[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    reinterpret_cast<uint4*>(x16 + size_t(t) * H)[p] = o;
    // planes: a 32-value block spans 4 lanes (8 values each)
    uint32_t am = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) am = max(am, __float_as_uint(f[i]) & 0x7FFFFFFFu);
    am = max(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = max(am, __shfl_xor_sync(0xffffffffu, am, 2));
    const int s = block_exp(am);
    uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint8_t hb, lb;
      split_e4m3(f[i], s, hb, lb);
      hw[i >> 2] |= uint32_t(hb) << (8 * (i & 3));
      lw[i >> 2] |= uint32_t(lb) << (8 * (i & 3));
    }
    const uint8_t eh = uint8_t(s + 127), el = uint8_t(max(1, s + 123));
    for (int j = 0; j < nd; ++j) {
      const size_t row = size_t(dst[j]);
      reinterpret_cast<uint2*>(xq_hi + row * H)[p] = make_uint2(hw[0], hw[1]);
      reinterpret_cast<uint2*>(xq_lo + row * H)[p] = make_uint2(lw[0], lw[1]);
      if ((lane & 3) == 0) {
        xs_hi[row * (H / 32) + p / 4] = eh;
        xs_lo[row * (H / 32) + p / 4] = el;
      }
    }
  }
}


// ------------------------------------------------------------------ GEMM

// Tile geometry shared by the roles.
struct MxGeo {
  int ebase;           // first weight row of the tile's expert (w13)
  int K, nk;           // reduction length and its 128-wide chunks
  int brow0;           // first activation row (slot) of the tile
  int n, n_load, n_mma;
  int wrow0, wrow1;    // first weight rows of the two 64-row halves
};

__device__ __forceinline__ MxGeo mx_geo(const MxParams& P, const MxTile& t, int brow0) {
  MxGeo g;
  g.n = t.n;
  g.n_load = (t.n + 31) / 32 * 32;
  g.n_mma = g.n_load;
  g.ebase = t.grp * 2 * P.I;
  if (P.mode == kMW13) {
    g.K = P.H;
    g.wrow0 = t.grp * 2 * P.I + t.row0;
    g.wrow1 = g.wrow0 + P.I;
  } else {
    g.K = P.I;
    g.wrow0 = t.grp * P.H + t.row0;
    g.wrow1 = g.wrow0 + 64;
  }
  g.nk = g.K / MBK;
  g.brow0 = brow0;
  return g;
}

// Instruction descriptor of kind::mxf8f6f4 with E2M1 A, E4M3 B, E8M0 scales,
// both operands K-major: A format bits 7-9 = 5, B format bits 10-12 = 0,
// N >> 3 at bits 17-22, scale format bit 23 = 1 (E8M0), M >> 4 at bits 24-28;
// the scale-factor byte ids (bits 4-5 for B, 29-30 for A) are set per K step.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N) {
  return (5u << 7) | (uint32_t(N >> 3) << 17) | (1u << 23) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void umma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc,
                                        uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(kMThreads, 1)
    k_mx_gemm(MxParams P, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBh,
              const __grid_constant__ CUtensorMap tmBl, const __grid_constant__ CUtensorMap tmSw,
              const __grid_constant__ CUtensorMap tmSh, const __grid_constant__ CUtensorMap tmSl) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int kMStages = P.nst, stage = mx_stage_bytes(P.bn);
  const int kMOffSc = kMStages * stage, slot = mx_scale_slot(P.bn);
  const int kMOffX = kMOffSc + 2 * slot;
  MxBars& B = *reinterpret_cast<MxBars*>(smem + kMOffX + kMXchBytes);
  TileCache& TC = *reinterpret_cast<TileCache*>(smem + kMOffX + kMXchBytes + kMBarBytes);
  volatile int* abort_flag = &B.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMStages; ++s) {
      mbar_init(&B.full[s], 1);
      mbar_init(&B.sf_full[s], 4);  // one arrival per scale-writer warp
      mbar_init(&B.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.acc_full[b], 1);
      mbar_init(&B.acc_empty[b], 4);  // one arrival per epilogue warp
      mbar_init(&B.sc_full[b], 1);
      mbar_init(&B.sc_empty[b], 4);   // one arrival per scale-writer warp
    }
    mbar_init(&B.done, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&B.tmem_base, kMTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;
  pdl_wait();  // tiles, routing and activations come from earlier kernels
  const int nmine = cache_tiles(P, *P.ntiles - P.shared_tiles, TC);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmBh);
    prefetch_tmap(&tmBl);
    prefetch_tmap(&tmSw);
    prefetch_tmap(&tmSh);
    prefetch_tmap(&tmSl);
    uint32_t gc = 0, gs = 0;
    bool ok = true;
    for (int li = 0; li < nmine && ok; ++li) {
      int brow0;
      const MxTile t = tile_at(P, TC, li, brow0);
      const MxGeo g = mx_geo(P, t, brow0);
      for (int c = 0; c < g.nk; ++c, ++gc) {
        if ((c & 3) == 0) {  // scales of this chunk and the next three
          const uint32_t j = gs & 1u, v = gs >> 1;
          if (!mwait(&B.sc_empty[j], (v & 1u) ^ 1u, abort_flag, P.status)) {
            ok = false;
            break;
          }
          char* sc = smem + kMOffSc + j * slot;
          mbar_arrive_expect_tx(&B.sc_full[j], uint32_t(16 * (MBM + 2 * g.n_load)));
          if (P.mode == kMW13)
            tma_load_3d(sc, &tmSw, c * 4, g.wrow0 - g.ebase, 2 * t.grp, &B.sc_full[j]);
          else
            tma_load_2d(sc, &tmSw, c * 4, g.wrow0, &B.sc_full[j]);
          for (int i = 0; i < g.n_load / 32; ++i) {
            tma_load_2d(sc + 16 * MBM + 512 * i, &tmSh, c * 4, g.brow0 + 32 * i, &B.sc_full[j]);
            tma_load_2d(sc + 16 * (MBM + P.bn) + 512 * i, &tmSl, c * 4, g.brow0 + 32 * i, &B.sc_full[j]);
          }
          ++gs;
        }
        const int s = gc % kMStages;
        const uint32_t u = gc / kMStages;
        if (!mwait(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        // E2M1 rows count their packed bytes (64 per row and chunk); the
        // activation planes come in boxes of 32 rows, as many as the tile's
        // tokens need (rows past them only feed columns the epilogue ignores).
        mbar_arrive_expect_tx(&B.full[s], uint32_t(MBM * MBK / 2 + 2 * g.n_load * MBK));
        char* as = smem + s * stage;
        if (P.mode == kMW13)  // gate and up halves in one box of the 3-D map
          tma_load_3d(as, &tmA, c * MBK, g.wrow0 - g.ebase, 2 * t.grp, &B.full[s]);
        else
          tma_load_2d(as, &tmA, c * MBK, g.wrow0, &B.full[s]);
        for (int i = 0; i < g.n_load / 32; ++i) {
          tma_load_2d(as + kMA + i * 32 * MBK, &tmBh, c * MBK, g.brow0 + 32 * i, &B.full[s]);
          tma_load_2d(as + kMA + P.bn * MBK + i * 32 * MBK, &tmBl, c * MBK, g.brow0 + 32 * i, &B.full[s]);
        }
      }
    }
    for (uint32_t q = 0; q < uint32_t(kMStages) && q < gc; ++q) {
      const uint32_t gq = gc - 1 - q;
      mbar_wait_bounded(&B.full[gq % kMStages], (gq / kMStages) & 1u, kMTries);
    }
    for (uint32_t q = 0; q < 2u && q < gs; ++q) {
      const uint32_t gq = gs - 1 - q;
      mbar_wait_bounded(&B.sc_full[gq & 1u], (gq >> 1) & 1u, kMTries);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t gc = 0, lt = 0;
    bool ok = true;
    for (int li = 0; li < nmine && ok; ++li, ++lt) {
      int brow0;
      const MxGeo g = mx_geo(P, tile_at(P, TC, li, brow0), brow0);
      const uint32_t b = lt & 1u, v = lt >> 1;
      if (!mwait(&B.acc_empty[b], (v & 1u) ^ 1u, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t d = tmem + b * MBN;
      const uint32_t idesc = idesc_mx(MBM, g.n_mma);
      for (int c = 0; c < g.nk; ++c, ++gc) {
        const int s = gc % kMStages;
        const uint32_t u = gc / kMStages;
        if (!mwait(&B.full[s], u & 1u, abort_flag, P.status) ||
            !mwait(&B.sf_full[s], u & 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * stage);
        const uint32_t bh0 = a0 + kMA;
        const uint32_t bl0 = bh0 + P.bn * MBK;
        const uint32_t sf = tmem + kMColSF + 12u * uint32_t(s);
#pragma unroll
        for (int kk = 0; kk < MBK / 32; ++kk) {
          const uint32_t id = idesc | (uint32_t(kk) << 29) | (uint32_t(kk) << 4);
          const uint32_t byte = uint32_t(kk) << 30;
          const uint64_t ad = sw128_kmajor_desc(a0 + kk * 32);
          umma_mx(d, ad, sw128_kmajor_desc(bh0 + kk * 32), id, (c > 0 || kk > 0) ? 1u : 0u, sf | byte,
                  (sf + 4) | byte);
          umma_mx(d, ad, sw128_kmajor_desc(bl0 + kk * 32), id, 1u, sf | byte, (sf + 8) | byte);
        }
        umma_commit(&B.empty[s]);
      }
      if (!ok) break;
      umma_commit(&B.acc_full[b]);
    }
    umma_commit(&B.done);
    mbar_wait_bounded(&B.done, 0, kMTries);
  } else if (warp >= 8) {
    // ------------------------------------------------------------ scale writers
    // The scales of four chunks arrive by TMA in a scale slot (a global load
    // here would wait behind the SM's copies in flight); per chunk each warp
    // moves its lane quarter's copy into TMEM.
    const int q = warp - 8;  // TMEM lane quarter of this warp (warp % 4)
    uint32_t gc = 0, gs = 0;
    bool ok = true;
    for (int li = 0; li < nmine && ok; ++li) {
      int brow0;
      const MxTile t = tile_at(P, TC, li, brow0);
      const MxGeo g = mx_geo(P, t, brow0);
      for (int c = 0; c < g.nk && ok; ++c, ++gc) {
        const uint32_t j = gs & 1u;
        if ((c & 3) == 0 && !__all_sync(0xffffffffu, mwait(&B.sc_full[j], (gs >> 1) & 1u, abort_flag, P.status))) {
          ok = false;
          break;
        }
        const int s = gc % kMStages;
        const uint32_t u = gc / kMStages;
        if (!__all_sync(0xffffffffu, mwait(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // row 32 i + lane of each operand, the four bytes of this chunk
        const char* sc = smem + kMOffSc + j * slot + 4 * (c & 3);
        uint32_t wa[4], hv[4], lv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 32 * i + lane;
          wa[i] = *reinterpret_cast<const uint32_t*>(sc + 16 * r);
          hv[i] = r < g.n_mma ? *reinterpret_cast<const uint32_t*>(sc + 16 * (MBM + r)) : 0u;
          lv[i] = r < g.n_mma ? *reinterpret_cast<const uint32_t*>(sc + 16 * (MBM + P.bn + r)) : 0u;
        }
        const uint32_t sf = tmem + kMColSF + 12u * uint32_t(s) + (uint32_t(32 * q) << 16);
        tmem_st_32x32b_x4(sf, wa[0], wa[1], wa[2], wa[3]);
        tmem_st_32x32b_x4(sf + 4, hv[0], hv[1], hv[2], hv[3]);
        tmem_st_32x32b_x4(sf + 8, lv[0], lv[1], lv[2], lv[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.sf_full[s]);
          if ((c & 3) == 3) mbar_arrive(&B.sc_empty[j]);
        }
        if ((c & 3) == 3) ++gs;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;  // TMEM lane quarter
    float* xch = reinterpret_cast<float*>(smem + kMOffX);
    uint32_t lt = 0;
    for (int li = 0; li < nmine; ++li, ++lt) {
      int brow0;
      const MxTile t = tile_at(P, TC, li, brow0);
      const MxGeo g = mx_geo(P, t, brow0);
      const uint32_t b = lt & 1u, v = lt >> 1;
      const int row = 32 * q + lane;
      const bool got = mwait(&B.acc_full[b], v & 1u, abort_flag, P.status);
      named_bar_sync(1, 128);
      if (!got || *abort_flag) break;
      tc_fence_after();
      const uint32_t acc = tmem + b * MBN + (uint32_t(32 * q) << 16);
      for (int c0 = 0; c0 < g.n; c0 += 32) {
        uint32_t rv[32];
        tmem_ld_32x32b_x32(acc + c0, rv);
        tmem_wait_ld();
        if (P.mode == kMW13) {
          // Lane quarters 0-1 hold the gate rows of channels 32 q + lane, 2-3
          // the up rows. Each quarter hands the other half of its columns to
          // its partner and finishes 16 columns: SwiGLU, then both E4M3 planes
          // of the 32-channel block (this warp's lanes) per token.
          const int part = q ^ 2;  // partner quarter (same channels)
          const int cbase = q < 2 ? 16 : 0;   // columns handed over
#pragma unroll
          for (int i = 0; i < 16; ++i) xch[(q * 32 + lane) * kMXch + i] = __uint_as_float(rv[cbase + i]);
          named_bar_sync(1, 128);
          const int ch = t.row0 + 32 * (q & 1) + lane;
          const int cown = q < 2 ? 0 : 16;     // columns finished here
#pragma unroll 4
          for (int i = 0; i < 16; ++i) {
            const int col = c0 + cown + i;
            if (col < g.n) {  // uniform across the warp
              const float mine = __uint_as_float(rv[cown + i]);
              const float other = xch[(part * 32 + lane) * kMXch + i];
              const float h = q < 2 ? clamped_swiglu_f(mine, other, P.limit) : clamped_swiglu_f(other, mine, P.limit);
              const uint32_t am = __reduce_max_sync(0xffffffffu, __float_as_uint(h) & 0x7FFFFFFFu);
              const int se = block_exp(am);
              uint8_t hb, lb;
              split_e4m3(h, se, hb, lb);
              const size_t slot = size_t(g.brow0 + col);
              P.h_hi[slot * P.I + ch] = hb;
              P.h_lo[slot * P.I + ch] = lb;
              if (lane == 0) {
                P.hs_hi[slot * (P.I / 32) + ch / 32] = uint8_t(se + 127);
                P.hs_lo[slot * (P.I / 32) + ch / 32] = uint8_t(max(1, se + 123));
              }
            }
          }
          named_bar_sync(1, 128);
        } else {
          const int m = t.row0 + row;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = c0 + i;
            if (col < g.n) P.y_slot[size_t(g.brow0 + col) * P.H + m] = __float2bfloat16_rn(__uint_as_float(rv[i]));
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
    tmem_dealloc(tmem, kMTmemCols);
  }
}

// ------------------------------------------------------------------ token-major GEMM
//
// For experts with many tokens the roles swap: a tile is 128 slots (MMA M, the
// activation planes as A) by 256 weight rows (MMA N, the E2M1 codes as B), so
// one 64 KB stage feeds eight M128 x N256 x K32 MMAs and the weight and
// activation chunks are each read once per tile. w13 tiles cover 128 channels
// (their gate rows, then their up rows: accumulator columns 0-127 and
// 128-255), w2 tiles 256 output rows. The scales also come through TMA, 16
// bytes (four chunks) per row at a time, into a two-slot ring; the scale
// warps move them into TMEM. With the operands swapped the epilogue is per
// thread: lane = slot, so the clamped SwiGLU, the 32-channel block scale and
// the two h planes need no exchange between threads.
//
//   warp 0       TMA producer (operand stages and scale slots)
//   warp 1       TMEM owner and MMA issuer
//   warps 2-5    scale writers (TMEM lane quarter = warp % 4)
//   warps 6-21   epilogue, four per lane quarter, each a quarter of the columns
constexpr int XM = 128, XN = 256, XK = 128;
constexpr int kXStages = 3;
constexpr int kXFirstEpi = 6;
constexpr int kXEpiWarps = 16;
constexpr int kXThreads = 32 * (kXFirstEpi + kXEpiWarps);
constexpr int kXA = XM * XK;            // 16 KB per activation plane
constexpr int kXB = XN * XK;            // 32 KB: the codes expanded to one byte each
constexpr int kXStage = 2 * kXA + kXB;  // 64 KB
constexpr int kXScW = 0;                // scale slot: 256 weight rows, 128 + 128 slot rows, 16 B each
constexpr int kXScH = XN * 16;
constexpr int kXScL = kXScH + XM * 16;
constexpr int kXSc = kXScL + XM * 16;   // 8 KB
constexpr int kXOffSc = kXStages * kXStage;
constexpr int kXOffBar = kXOffSc + 2 * kXSc;
constexpr int kXOffTiles = kXOffBar + 256;
constexpr int kXSmem = kXOffTiles + kTileCacheBytes + 1024;
static_assert(kXSmem <= kMSmemMax, "dynamic shared memory per block");
constexpr uint32_t kXColSF = XN;        // per stage 16 columns: SFA hi (4), SFA lo (4), SFB (8)
constexpr uint32_t kXTmemCols = 512;

struct XBars {
  uint64_t full[kXStages];
  uint64_t empty[kXStages];
  uint64_t sf_full[kXStages];
  uint64_t sc_full[2];
  uint64_t sc_empty[2];
  uint64_t acc_full, acc_empty, done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(XBars) <= 256, "barrier block");

struct XGeo {
  int K, nk;     // reduction length and its chunks of XK
  int brow0, n;  // first slot and slot count of the tile
  int wy, wz;    // weight coordinates: w13 (channel, 2 expert), w2 (row, unused)
};

__device__ __forceinline__ XGeo xgeo(const MxParams& P, const MxTile& t, int brow0) {
  XGeo g;
  g.n = t.n;
  g.brow0 = brow0;
  if (P.mode == kMW13) {
    g.K = P.H;
    g.wy = t.row0;
    g.wz = 2 * t.grp;
  } else {
    g.K = P.I;
    g.wy = t.grp * P.H + t.row0;
    g.wz = 0;
  }
  g.nk = g.K / XK;
  return g;
}

// kind::mxf8f6f4 with E4M3 A (activations) and E2M1 B (weights).
__host__ __device__ constexpr uint32_t idesc_mxt(int M, int N) {
  return (0u << 7) | (5u << 10) | (uint32_t(N >> 3) << 17) | (1u << 23) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__global__ void __launch_bounds__(kXThreads, 1)
    k_mxt_gemm(MxParams P, const __grid_constant__ CUtensorMap tmAh, const __grid_constant__ CUtensorMap tmAl,
               const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmSw,
               const __grid_constant__ CUtensorMap tmSh, const __grid_constant__ CUtensorMap tmSl) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  XBars& B = *reinterpret_cast<XBars*>(smem + kXOffBar);
  TileCache& TC = *reinterpret_cast<TileCache*>(smem + kXOffTiles);
  volatile int* abort_flag = &B.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool w13 = P.mode == kMW13;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&B.full[s], 1);
      mbar_init(&B.empty[s], 1);
      mbar_init(&B.sf_full[s], 4);  // one arrival per scale warp
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&B.sc_full[j], 1);
      mbar_init(&B.sc_empty[j], 4);
    }
    mbar_init(&B.acc_full, 1);
    mbar_init(&B.acc_empty, kXEpiWarps);
    mbar_init(&B.done, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&B.tmem_base, kXTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;
  pdl_wait();  // tiles, routing and activations come from earlier kernels
  const int nmine = cache_tiles(P, *P.ntiles - P.shared_tiles, TC);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_tmap(&tmAh);
    prefetch_tmap(&tmAl);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSw);
    prefetch_tmap(&tmSh);
    prefetch_tmap(&tmSl);
    uint32_t gc = 0, gs = 0;
    bool ok = true;
    for (int li = 0; li < nmine && ok; ++li) {
      int brow0;
      const XGeo g = xgeo(P, tile_at(P, TC, li, brow0), brow0);
      for (int c = 0; c < g.nk; ++c, ++gc) {
        if ((c & 3) == 0) {  // scales of this chunk and the next three
          const uint32_t j = gs & 1u, v = gs >> 1;
          if (!mwait(&B.sc_empty[j], (v & 1u) ^ 1u, abort_flag, P.status)) {
            ok = false;
            break;
          }
          char* sc = smem + kXOffSc + j * kXSc;
          mbar_arrive_expect_tx(&B.sc_full[j], uint32_t(kXSc));
          if (w13)
            tma_load_3d(sc + kXScW, &tmSw, c * 4, g.wy, g.wz, &B.sc_full[j]);
          else
            tma_load_2d(sc + kXScW, &tmSw, c * 4, g.wy, &B.sc_full[j]);
          tma_load_2d(sc + kXScH, &tmSh, c * 4, g.brow0, &B.sc_full[j]);
          tma_load_2d(sc + kXScL, &tmSl, c * 4, g.brow0, &B.sc_full[j]);
          ++gs;
        }
        const int s = gc % kXStages;
        const uint32_t u = gc / kXStages;
        if (!mwait(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        // E2M1 rows count their packed bytes (64 per row and chunk)
        mbar_arrive_expect_tx(&B.full[s], uint32_t(2 * kXA + XN * XK / 2));
        char* st = smem + s * kXStage;
        tma_load_2d(st, &tmAh, c * XK, g.brow0, &B.full[s]);
        tma_load_2d(st + kXA, &tmAl, c * XK, g.brow0, &B.full[s]);
        if (w13)  // gate and up rows of 128 channels in one box of the 3-D map
          tma_load_3d(st + 2 * kXA, &tmB, c * XK, g.wy, g.wz, &B.full[s]);
        else
          tma_load_2d(st + 2 * kXA, &tmB, c * XK, g.wy, &B.full[s]);
      }
    }
    // nothing may still be landing in shared memory when the CTA exits
    for (uint32_t q = 0; q < uint32_t(kXStages) && q < gc; ++q) {
      const uint32_t gq = gc - 1 - q;
      mbar_wait_bounded(&B.full[gq % kXStages], (gq / kXStages) & 1u, kMTries);
    }
    for (uint32_t q = 0; q < 2u && q < gs; ++q) {
      const uint32_t gq = gs - 1 - q;
      mbar_wait_bounded(&B.sc_full[gq & 1u], (gq >> 1) & 1u, kMTries);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t gc = 0, lt = 0;
    bool ok = true;
    const uint32_t idesc = idesc_mxt(XM, XN);
    for (int li = 0; li < nmine && ok; ++li, ++lt) {
      int brow0;
      const XGeo g = xgeo(P, tile_at(P, TC, li, brow0), brow0);
      if (!mwait(&B.acc_empty, (lt & 1u) ^ 1u, abort_flag, P.status)) break;
      tc_fence_after();
      for (int c = 0; c < g.nk; ++c, ++gc) {
        const int s = gc % kXStages;
        const uint32_t u = gc / kXStages;
        if (!mwait(&B.full[s], u & 1u, abort_flag, P.status) ||
            !mwait(&B.sf_full[s], u & 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ah = smem_u32(smem + s * kXStage);
        const uint32_t al = ah + kXA;
        const uint32_t bw = ah + 2 * kXA;
        const uint32_t sf = tmem + kXColSF + 16u * uint32_t(s);
#pragma unroll
        for (int kk = 0; kk < XK / 32; ++kk) {
          const uint32_t id = idesc | (uint32_t(kk) << 29) | (uint32_t(kk) << 4);
          const uint32_t byte = uint32_t(kk) << 30;
          const uint64_t bd = sw128_kmajor_desc(bw + kk * 32);
          umma_mx(tmem, sw128_kmajor_desc(ah + kk * 32), bd, id, (c > 0 || kk > 0) ? 1u : 0u, sf | byte,
                  (sf + 8) | byte);
          umma_mx(tmem, sw128_kmajor_desc(al + kk * 32), bd, id, 1u, (sf + 4) | byte, (sf + 8) | byte);
        }
        umma_commit(&B.empty[s]);
      }
      if (!ok) break;
      umma_commit(&B.acc_full);
    }
    umma_commit(&B.done);
    mbar_wait_bounded(&B.done, 0, kMTries);
  } else if (warp >= 2 && warp < kXFirstEpi) {
    // ------------------------------------------------------------ scale writers
    // Lane l of every lane quarter holds operand row 32 i + l in column i, one
    // byte per K step: columns 0-3 the slots' hi scales, 4-7 their lo scales,
    // 8-15 the 256 weight rows.
    const int q = warp & 3;
    uint32_t gc = 0, gs = 0;
    bool ok = true;
    for (int li = 0; li < nmine && ok; ++li) {
      int brow0;
      const XGeo g = xgeo(P, tile_at(P, TC, li, brow0), brow0);
      for (int c = 0; c < g.nk && ok; ++c, ++gc) {
        const uint32_t j = gs & 1u;
        if ((c & 3) == 0 && !__all_sync(0xffffffffu, mwait(&B.sc_full[j], (gs >> 1) & 1u, abort_flag, P.status))) {
          ok = false;
          break;
        }
        const int s = gc % kXStages;
        const uint32_t u = gc / kXStages;
        if (!__all_sync(0xffffffffu, mwait(&B.empty[s], (u & 1u) ^ 1u, abort_flag, P.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const char* sc = smem + kXOffSc + j * kXSc + 4 * (c & 3);
        uint32_t wv[8], hv[4], lv[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) wv[i] = *reinterpret_cast<const uint32_t*>(sc + kXScW + (32 * i + lane) * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          hv[i] = *reinterpret_cast<const uint32_t*>(sc + kXScH + (32 * i + lane) * 16);
          lv[i] = *reinterpret_cast<const uint32_t*>(sc + kXScL + (32 * i + lane) * 16);
        }
        const uint32_t ta = tmem + kXColSF + 16u * uint32_t(s) + (uint32_t(32 * q) << 16);
        tmem_st_32x32b_x4(ta, hv[0], hv[1], hv[2], hv[3]);
        tmem_st_32x32b_x4(ta + 4, lv[0], lv[1], lv[2], lv[3]);
        tmem_st_32x32b_x8(ta + 8, wv);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.sf_full[s]);
          if ((c & 3) == 3) mbar_arrive(&B.sc_empty[j]);
        }
        if ((c & 3) == 3) ++gs;
      }
    }
  } else if (warp >= kXFirstEpi) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter
    const int sub = (warp - kXFirstEpi) >> 2;  // quarter of the columns
    const int row = 32 * q + lane;
    uint32_t lt = 0;
    for (int li = 0; li < nmine; ++li, ++lt) {
      int brow0;
      const MxTile t = tile_at(P, TC, li, brow0);
      const XGeo g = xgeo(P, t, brow0);
      if (!__all_sync(0xffffffffu, mwait(&B.acc_full, lt & 1u, abort_flag, P.status)) || *abort_flag) break;
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t(32 * q) << 16);
      const bool valid = row < g.n;
      const size_t slot = size_t(g.brow0 + row);
      if (w13) {
        // columns 32 sub .. +31 (gate) and 128 + 32 sub .. (up): one 32-channel block
        uint32_t gr[32], ur[32];
        tmem_ld_32x32b_x32(acc + 32 * sub, gr);
        tmem_ld_32x32b_x32(acc + XN / 2 + 32 * sub, ur);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.acc_empty);
        if (valid) {
          uint32_t am = 0;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float h = clamped_swiglu_f(__uint_as_float(gr[i]), __uint_as_float(ur[i]), P.limit);
            gr[i] = __float_as_uint(h);
            am = max(am, gr[i] & 0x7FFFFFFFu);
          }
          const int se = block_exp(am);
          uint32_t hw[8], lw[8];
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            hw[w] = 0u;
            lw[w] = 0u;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              uint8_t hb, lb;
              split_e4m3(__uint_as_float(gr[4 * w + b]), se, hb, lb);
              hw[w] |= uint32_t(hb) << (8 * b);
              lw[w] |= uint32_t(lb) << (8 * b);
            }
          }
          const int ch = t.row0 + 32 * sub;
          uint4* dh = reinterpret_cast<uint4*>(P.h_hi + slot * P.I + ch);
          uint4* dl = reinterpret_cast<uint4*>(P.h_lo + slot * P.I + ch);
          dh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          dh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
          dl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          dl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
          P.hs_hi[slot * (P.I / 32) + ch / 32] = uint8_t(se + 127);
          P.hs_lo[slot * (P.I / 32) + ch / 32] = uint8_t(max(1, se + 123));
        }
      } else {
        // columns 64 sub .. +63 of the 256 output rows
        uint32_t ya[32], yb[32];
        tmem_ld_32x32b_x32(acc + 64 * sub, ya);
        tmem_ld_32x32b_x32(acc + 64 * sub + 32, yb);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.acc_empty);
        if (valid) {
          uint4* dy = reinterpret_cast<uint4*>(P.y_slot + slot * P.H + t.row0 + 64 * sub);
          auto pk = [](uint32_t a, uint32_t b) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(a), __uint_as_float(b));
            return *reinterpret_cast<const uint32_t*>(&v);
          };
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dy[i] = make_uint4(pk(ya[8 * i], ya[8 * i + 1]), pk(ya[8 * i + 2], ya[8 * i + 3]),
                               pk(ya[8 * i + 4], ya[8 * i + 5]), pk(ya[8 * i + 6], ya[8 * i + 7]));
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dy[4 + i] = make_uint4(pk(yb[8 * i], yb[8 * i + 1]), pk(yb[8 * i + 2], yb[8 * i + 3]),
                                   pk(yb[8 * i + 4], yb[8 * i + 5]), pk(yb[8 * i + 6], yb[8 * i + 7]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kXTmemCols);
  }
}


// 3-D map of the w13 codes: {K, I rows of a half, 2 E halves}; box {128, 64, 2}
// brings a tile's 64 gate rows and the matching 64 up rows in one copy.
bool mx_map_w13(CUtensorMap* m, const void* base, uint64_t K, uint64_t I, uint64_t halves) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[3] = {K, I, halves};
  const cuuint64_t strides[2] = {K / 2, I * (K / 2)};
  const cuuint32_t box[3] = {128, 64, 2};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map, 128-byte swizzle, box {128 elements, box_rows}.
bool mx_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t row_bytes, uint64_t rows,
            uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  if (rows == 0) rows = 1;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// General 2-D / 3-D maps ([halves][rows][cols], rows row_bytes apart).
bool mx_map2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t row_bytes, uint64_t rows,
              uint32_t bx, uint32_t by, CUtensorMapSwizzle sw) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  if (rows == 0) rows = 1;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {bx, by};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool mx_map3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t row_bytes, uint64_t rows,
              uint64_t halves, uint32_t bx, uint32_t by, CUtensorMapSwizzle sw) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cols, rows, halves};
  const cuuint64_t strides[2] = {row_bytes, rows * row_bytes};
  const cuuint32_t box[3] = {bx, by, 2};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool mx_supported(const v4moe_config& c, const v4moe_weights& w) {
  auto a32 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; };
  return c.hidden % 512 == 0 && c.inter % 512 == 0 && a32(w.w13_codes) && a32(w.w2_codes) &&
         (reinterpret_cast<uintptr_t>(w.w13_scales) & 15) == 0 && (reinterpret_cast<uintptr_t>(w.w2_scales) & 15) == 0 &&
         tensor_map_encoder() != nullptr;
}

cudaError_t launch_mx_gather(const ForwardArgs& a, __half* x16, int* sigma, const MxBuffers& m, cudaStream_t st) {
  const v4moe_config& c = a.c;
  return launch_kernel("mx_gather", k_mx_gather, dim3((a.T + 7) / 8), dim3(256), 0, st, false, a.T, c.hidden,
                       c.n_experts, c.top_k, a.x, a.topk_ids, a.slot_pos, x16, sigma, m.xq_hi, m.xq_lo, m.xs_hi,
                       m.xs_lo);
}

cudaError_t launch_mx_gemm(const ForwardArgs& a, int w2, const void* tiles, const int* ntiles, int shared_tiles,
                           int bn, const MxBuffers& m, cudaStream_t st) {
  const v4moe_config& c = a.c;
  const int64_t S = int64_t(a.T) * c.top_k;
  MxParams P;
  P.T = a.T;
  P.H = c.hidden;
  P.I = c.inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.limit = c.swiglu_limit;
  P.mode = w2 ? kMW2 : kMW13;
  P.offsets = a.offsets;
  P.tiles = static_cast<const MxTile*>(tiles);
  P.ntiles = ntiles;
  P.shared_tiles = shared_tiles;
  P.h_hi = m.hq_hi;
  P.h_lo = m.hq_lo;
  P.hs_hi = m.hs_hi;
  P.hs_lo = m.hs_lo;
  P.y_slot = a.y_slot;
  P.status = a.status;
  CUtensorMap mA, mBh, mBl, mSw, mSh, mSl;
  bool ok = true;
  constexpr auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  constexpr auto NS = CU_TENSOR_MAP_SWIZZLE_NONE;
  const uint64_t H = c.hidden, I = c.inter, E = c.n_experts;
  if (!w2) {
    P.w_scales = a.w.w13_scales;
    P.b_sc_hi = m.xs_hi;
    P.b_sc_lo = m.xs_lo;
    ok &= mx_map3d(&mSw, a.w.w13_scales, U8, H / 32, H / 32, I, 2 * E, 16, MBM / 2, NS);
    ok &= mx_map2d(&mSh, m.xs_hi, U8, H / 32, H / 32, S, 16, 32, NS);
    ok &= mx_map2d(&mSl, m.xs_lo, U8, H / 32, H / 32, S, 16, 32, NS);
    ok &= mx_map_w13(&mA, a.w.w13_codes, c.hidden, c.inter, uint64_t(c.n_experts) * 2);
    ok &= mx_map(&mBh, m.xq_hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.hidden, c.hidden, S, 32);
    ok &= mx_map(&mBl, m.xq_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.hidden, c.hidden, S, 32);
  } else {
    P.w_scales = a.w.w2_scales;
    P.b_sc_hi = m.hs_hi;
    P.b_sc_lo = m.hs_lo;
    ok &= mx_map2d(&mSw, a.w.w2_scales, U8, I / 32, I / 32, E * H, 16, MBM, NS);
    ok &= mx_map2d(&mSh, m.hs_hi, U8, I / 32, I / 32, S, 16, 32, NS);
    ok &= mx_map2d(&mSl, m.hs_lo, U8, I / 32, I / 32, S, 16, 32, NS);
    ok &= mx_map(&mA, a.w.w2_codes, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, c.inter, c.inter / 2,
                 uint64_t(c.n_experts) * c.hidden, MBM);
    ok &= mx_map(&mBh, m.hq_hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.inter, c.inter, S, 32);
    ok &= mx_map(&mBl, m.hq_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.inter, c.inter, S, 32);
  }
  if (!ok) return cudaErrorInvalidValue;
  const int sms = device_sms();
  // as many stages as fit next to the epilogue exchange and the barriers
  P.bn = bn;
  const int fixed = 2 * mx_scale_slot(bn) + kMXchBytes + kMBarBytes + kTileCacheBytes + 1024;
  P.nst = std::min(kMMaxStages, (kMSmemMax - fixed) / mx_stage_bytes(bn));
  const int smem = P.nst * mx_stage_bytes(bn) + fixed;
  set_smem(k_mx_gemm, smem);
  return launch_kernel(w2 ? "mx_w2" : "mx_w13", k_mx_gemm, dim3(sms), dim3(kMThreads), smem, st, true, P, mA, mBh,
                       mBl, mSw, mSh, mSl);
}

cudaError_t launch_mxt_gemm(const ForwardArgs& a, int w2, const void* tiles, const int* ntiles, int shared_tiles,
                            const MxBuffers& m, cudaStream_t st) {
  const v4moe_config& c = a.c;
  const uint64_t S = uint64_t(a.T) * c.top_k;
  const uint64_t H = c.hidden, I = c.inter, E = c.n_experts;
  MxParams P;
  P.T = a.T;
  P.H = c.hidden;
  P.I = c.inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.limit = c.swiglu_limit;
  P.mode = w2 ? kMW2 : kMW13;
  P.offsets = a.offsets;
  P.tiles = static_cast<const MxTile*>(tiles);
  P.ntiles = ntiles;
  P.shared_tiles = shared_tiles;
  P.h_hi = m.hq_hi;
  P.h_lo = m.hq_lo;
  P.hs_hi = m.hs_hi;
  P.hs_lo = m.hs_lo;
  P.y_slot = a.y_slot;
  P.status = a.status;
  P.w_scales = nullptr;
  P.b_sc_hi = nullptr;
  P.b_sc_lo = nullptr;
  constexpr auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  constexpr auto U4 = CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
  constexpr auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  constexpr auto NS = CU_TENSOR_MAP_SWIZZLE_NONE;
  CUtensorMap mAh, mAl, mB, mSw, mSh, mSl;
  bool ok = true;
  if (!w2) {
    ok &= mx_map2d(&mAh, m.xq_hi, U8, H, H, S, XK, XM, SW);
    ok &= mx_map2d(&mAl, m.xq_lo, U8, H, H, S, XK, XM, SW);
    ok &= mx_map3d(&mB, a.w.w13_codes, U4, H, H / 2, I, 2 * E, XK, XN / 2, SW);
    ok &= mx_map3d(&mSw, a.w.w13_scales, U8, H / 32, H / 32, I, 2 * E, 16, XN / 2, NS);
    ok &= mx_map2d(&mSh, m.xs_hi, U8, H / 32, H / 32, S, 16, XM, NS);
    ok &= mx_map2d(&mSl, m.xs_lo, U8, H / 32, H / 32, S, 16, XM, NS);
  } else {
    ok &= mx_map2d(&mAh, m.hq_hi, U8, I, I, S, XK, XM, SW);
    ok &= mx_map2d(&mAl, m.hq_lo, U8, I, I, S, XK, XM, SW);
    ok &= mx_map2d(&mB, a.w.w2_codes, U4, I, I / 2, E * H, XK, XN, SW);
    ok &= mx_map2d(&mSw, a.w.w2_scales, U8, I / 32, I / 32, E * H, 16, XN, NS);
    ok &= mx_map2d(&mSh, m.hs_hi, U8, I / 32, I / 32, S, 16, XM, NS);
    ok &= mx_map2d(&mSl, m.hs_lo, U8, I / 32, I / 32, S, 16, XM, NS);
  }
  if (!ok) return cudaErrorInvalidValue;
  const int sms = device_sms();
  set_smem(k_mxt_gemm, kXSmem);
  return launch_kernel(w2 ? "mxt_w2" : "mxt_w13", k_mxt_gemm, dim3(sms), dim3(kXThreads), kXSmem, st, true, P, mAh,
                       mAl, mB, mSw, mSh, mSl);
}

}  // namespace v4moe
