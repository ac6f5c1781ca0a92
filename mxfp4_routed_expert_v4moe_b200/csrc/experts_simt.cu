// Grouped expert GEMV/GEMM on CUDA cores (fp32 FMA), the general fallback of
// the expert computation for any token count, and the reference structure the
// tensor-core paths are measured against.
//
// Per group (routed expert e, or the shared expert):
//   w13 step:  [g; u] = W13 x_t, h_t = silu(min(g, L)) * clamp(u, -L, L)
//              ("Checked in its code" row "SwiGLU feed-forward"), h stored bf16
//   w2 step:   y_t = W2 h_t (fp32)
//   combine:   out[t] = bf16( sum_j w[t, j] * y_{slot(t, j)} + y_shared[t] )
// Routed weights are MXFP4 ("config.json" experts_w4a16: 4-bit float, group 32,
// e8m0 scale); shared weights are int8 per output channel (linears_w8a16).
//
// Layout of the work: CTA = (block of 32 output channels, group); the group's
// token rows are walked in chunks of kTok tokens staged as fp32 in shared
// memory; each warp owns 8 channels and lanes split K into 8-element pieces.
#include "launch.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kTok = 4;        // token rows per staged chunk
constexpr int kChanPerWarp = 8;
constexpr int kWarps = 4;
constexpr int kChanPerCta = kChanPerWarp * kWarps;

enum Fmt { kMx = 0, kInt8 = 1 };

// E2M1 code (0..15) -> fp32. The 3 magnitude bits are placed in the fp32
// exponent/mantissa so that the bit pattern is the code's value times 2^-126
// (code 1 lands on the subnormal 2^-127); one exact multiply by 2^126 restores
// it.
__device__ __forceinline__ float e2m1_f(uint32_t c) {
  return __uint_as_float(((c & 7u) << 22) | ((c & 8u) << 28)) * 0x1p126f;
}

// E8M0 byte -> 2^(e-127) as fp32 (e = 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_f(uint32_t e) {
  return e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);
}

// Dot of 8 weights (piece p of a row) with kTok staged activation rows.
template <int FMT>
struct Row;

template <>
struct Row<kMx> {
  const uint32_t* codes;  // 8 codes per u32
  const uint8_t* scales;  // one per 32 elements
  __device__ __forceinline__ Row(const uint8_t* c, const uint8_t* s, const float*)
      : codes(reinterpret_cast<const uint32_t*>(c)), scales(s) {}
  __device__ __forceinline__ void piece(int p, float w[8], float& sc) const {
    const uint32_t q = __ldg(codes + p);
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = e2m1_f((q >> (4 * i)) & 15u);
    sc = e8m0_f(__ldg(scales + (p >> 2)));
  }
  __device__ __forceinline__ float row_scale() const { return 1.0f; }
};

template <>
struct Row<kInt8> {
  const uint2* q;
  float s;
  __device__ __forceinline__ Row(const uint8_t* c, const uint8_t*, const float* rs)
      : q(reinterpret_cast<const uint2*>(c)), s(__ldg(rs)) {}
  __device__ __forceinline__ void piece(int p, float w[8], float& sc) const {
    const uint2 v = __ldg(q + p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w[i] = float(int8_t((v.x >> (8 * i)) & 0xFF));
      w[4 + i] = float(int8_t((v.y >> (8 * i)) & 0xFF));
    }
    sc = 1.0f;
  }
  __device__ __forceinline__ float row_scale() const { return s; }
};

template <int FMT>
__device__ __forceinline__ void row_dot(const Row<FMT>& row, int K, const float* xs, float acc[kTok]) {
  const int lane = threadIdx.x & 31;
  for (int p = lane; p < K / 8; p += 32) {
    float w[8], sc;
    row.piece(p, w, sc);
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
      const float4 a = *reinterpret_cast<const float4*>(xs + size_t(t) * K + 8 * p);
      const float4 b = *reinterpret_cast<const float4*>(xs + size_t(t) * K + 8 * p + 4);
      float part = w[0] * a.x;
      part = fmaf(w[1], a.y, part);
      part = fmaf(w[2], a.z, part);
      part = fmaf(w[3], a.w, part);
      part = fmaf(w[4], b.x, part);
      part = fmaf(w[5], b.y, part);
      part = fmaf(w[6], b.z, part);
      part = fmaf(w[7], b.w, part);
      acc[t] = fmaf(part, sc, acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    acc[t] *= row.row_scale();
  }
}

struct GroupParams {
  int T, H, I, Is, E, k;
  float limit;
  const __nv_bfloat16* x;
  const int32_t* offsets;
  const int32_t* sorted_slot;
  // routed weights
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  // shared weights
  const int8_t* sh13;
  const float* sh13_scale;
  const int8_t* sh2;
  const float* sh2_scale;
  __nv_bfloat16* h;
  float* y_slot;
  __nv_bfloat16* hs;
  float* ys;
};

// Stage rows [r, r + kTok) of the group (bf16 source rows) into xs as fp32.
__device__ __forceinline__ void stage_rows(float* xs, int K, int r, int nrows, const __nv_bfloat16* src,
                                           const int32_t* row_token, int kdiv, int row_base) {
  const int pieces = K / 8;
  for (int i = threadIdx.x; i < kTok * pieces; i += blockDim.x) {
    const int t = i / pieces, p = i % pieces;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (r + t < nrows) {
      const int row = row_token ? __ldg(row_token + row_base + r + t) / kdiv : row_base + r + t;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + size_t(row) * K) + p);
      a = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
      b = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
    }
    *reinterpret_cast<float4*>(xs + size_t(t) * K + 8 * p) = a;
    *reinterpret_cast<float4*>(xs + size_t(t) * K + 8 * p + 4) = b;
  }
}

template <int FMT>
__device__ void w13_group(const GroupParams& P, int Ig, int r_base, int nrows, const uint8_t* codes,
                          const uint8_t* scales, const float* rscale, const int32_t* row_token,
                          __nv_bfloat16* hout, float* xs) {
  const int H = P.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_bytes = FMT == kMx ? size_t(H) / 2 : size_t(H);
  const size_t srow_bytes = FMT == kMx ? size_t(H) / 32 : 0;
  for (int r = 0; r < nrows; r += kTok) {
    __syncthreads();
    stage_rows(xs, H, r, nrows, P.x, row_token, P.k, r_base);
    __syncthreads();
    for (int ch = 0; ch < kChanPerWarp; ++ch) {
      const int j = blockIdx.x * kChanPerCta + warp * kChanPerWarp + ch;
      if (j >= Ig) break;
      float g[kTok] = {}, u[kTok] = {};
      const Row<FMT> rg(codes + size_t(j) * row_bytes, scales + size_t(j) * srow_bytes, rscale + j);
      const Row<FMT> ru(codes + size_t(Ig + j) * row_bytes, scales + size_t(Ig + j) * srow_bytes,
                        rscale + Ig + j);
      row_dot<FMT>(rg, H, xs, g);
      row_dot<FMT>(ru, H, xs, u);
      if (lane < kTok && r + lane < nrows) {
        float gv = 0.f, uv = 0.f;
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t == lane) {
            gv = g[t];
            uv = u[t];
          }
        hout[size_t(r_base + r + lane) * Ig + j] = __float2bfloat16_rn(clamped_swiglu_f(gv, uv, P.limit));
      }
    }
  }
}

template <int FMT>
__device__ void w2_group(const GroupParams& P, int K, int r_base, int nrows, const uint8_t* codes,
                         const uint8_t* scales, const float* rscale, const __nv_bfloat16* hin,
                         float* yout, float* xs) {
  const int H = P.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_bytes = FMT == kMx ? size_t(K) / 2 : size_t(K);
  const size_t srow_bytes = FMT == kMx ? size_t(K) / 32 : 0;
  for (int r = 0; r < nrows; r += kTok) {
    __syncthreads();
    stage_rows(xs, K, r, nrows, hin, nullptr, 1, r_base);
    __syncthreads();
    for (int ch = 0; ch < kChanPerWarp; ++ch) {
      const int m = blockIdx.x * kChanPerCta + warp * kChanPerWarp + ch;
      if (m >= H) break;
      float acc[kTok] = {};
      const Row<FMT> row(codes + size_t(m) * row_bytes, scales + size_t(m) * srow_bytes, rscale + m);
      row_dot<FMT>(row, K, xs, acc);
      if (lane < kTok && r + lane < nrows) {
        float v = 0.f;
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t == lane) v = acc[t];
        yout[size_t(r_base + r + lane) * H + m] = v;
      }
    }
  }
}

__global__ void __launch_bounds__(kWarps * 32) k_w13_simt(GroupParams P) {
  extern __shared__ __align__(16) float xs[];
  const int g = blockIdx.y;
  if (g < P.E) {
    if (blockIdx.x * kChanPerCta >= P.I) return;
    const int r0 = P.offsets[g], n = P.offsets[g + 1] - r0;
    if (n <= 0) return;
    const size_t ecodes = size_t(2) * P.I * (P.H / 2), escales = size_t(2) * P.I * (P.H / 32);
    w13_group<kMx>(P, P.I, r0, n, P.w13_codes + g * ecodes, P.w13_scales + g * escales, nullptr,
                   P.sorted_slot, P.h, xs);
  } else {
    if (blockIdx.x * kChanPerCta >= P.Is) return;
    w13_group<kInt8>(P, P.Is, 0, P.T, reinterpret_cast<const uint8_t*>(P.sh13), nullptr, P.sh13_scale,
                     nullptr, P.hs, xs);
  }
}

__global__ void __launch_bounds__(kWarps * 32) k_w2_simt(GroupParams P) {
  extern __shared__ __align__(16) float xs[];
  const int g = blockIdx.y;
  if (blockIdx.x * kChanPerCta >= P.H) return;
  if (g < P.E) {
    const int r0 = P.offsets[g], n = P.offsets[g + 1] - r0;
    if (n <= 0) return;
    const size_t ecodes = size_t(P.H) * (P.I / 2), escales = size_t(P.H) * (P.I / 32);
    w2_group<kMx>(P, P.I, r0, n, P.w2_codes + g * ecodes, P.w2_scales + g * escales, nullptr, P.h,
                  P.y_slot, xs);
  } else {
    w2_group<kInt8>(P, P.Is, 0, P.T, reinterpret_cast<const uint8_t*>(P.sh2), nullptr, P.sh2_scale,
                    P.hs, P.ys, xs);
  }
}

// out[t] = bf16(sum_j w[t,j] * y_slot[slot_pos[t*k+j]] + ys[t]), j in order.
__global__ void __launch_bounds__(256) k_combine(int T, int H, int E, int k, const int32_t* __restrict__ ids,
                                                 const float* __restrict__ w, const int32_t* __restrict__ slot_pos,
                                                 const float* __restrict__ y_slot, const float* __restrict__ ys,
                                                 __nv_bfloat16* __restrict__ out) {
  const int t = blockIdx.x;
  for (int m = threadIdx.x * 4; m < H; m += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int e = ids[size_t(t) * k + j];
      if (e < 0 || e >= E) continue;
      const float wj = w[size_t(t) * k + j];
      const float4 y = *reinterpret_cast<const float4*>(y_slot + size_t(slot_pos[size_t(t) * k + j]) * H + m);
      acc.x = fmaf(wj, y.x, acc.x);
      acc.y = fmaf(wj, y.y, acc.y);
      acc.z = fmaf(wj, y.z, acc.z);
      acc.w = fmaf(wj, y.w, acc.w);
    }
    if (ys) {
      const float4 s = *reinterpret_cast<const float4*>(ys + size_t(t) * H + m);
      acc.x += s.x;
      acc.y += s.y;
      acc.z += s.z;
      acc.w += s.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + size_t(t) * H + m) = v;
  }
}

}  // namespace

cudaError_t launch_combine(const ForwardArgs& a, cudaStream_t st) {
  const v4moe_config& c = a.c;
  return launch_kernel("combine", k_combine, dim3(a.T), dim3(256), 0, st, false, a.T, c.hidden, c.n_experts,
                       c.top_k, a.topk_ids, a.topk_w, a.slot_pos, (const float*)a.y_slot,
                       (const float*)(c.shared_inter > 0 ? a.ys : nullptr), a.out);
}

cudaError_t launch_forward_simt(const ForwardArgs& a, cudaStream_t st) {
  const v4moe_config& c = a.c;
  if (a.T == 0) return cudaSuccess;
  GroupParams P;
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
  P.w13_codes = a.w.w13_codes;
  P.w13_scales = a.w.w13_scales;
  P.w2_codes = a.w.w2_codes;
  P.w2_scales = a.w.w2_scales;
  P.sh13 = a.w.sh_w13;
  P.sh13_scale = a.w.sh_w13_scale;
  P.sh2 = a.w.sh_w2;
  P.sh2_scale = a.w.sh_w2_scale;
  P.h = a.h;
  P.y_slot = a.y_slot;
  P.hs = a.hs;
  P.ys = a.ys;
  const int groups = c.n_experts + (c.shared_inter > 0 ? 1 : 0);
  const int maxI = c.shared_inter > c.inter ? c.shared_inter : c.inter;
  const size_t smem13 = size_t(kTok) * c.hidden * 4;
  const size_t smem2 = size_t(kTok) * maxI * 4;
  set_smem(k_w13_simt, smem13);
  set_smem(k_w2_simt, smem2);
  cudaError_t e = launch_kernel("w13_simt", k_w13_simt, dim3((maxI + kChanPerCta - 1) / kChanPerCta, groups),
                                dim3(kWarps * 32), smem13, st, false, P);
  if (e != cudaSuccess) return e;
  e = launch_kernel("w2_simt", k_w2_simt, dim3((c.hidden + kChanPerCta - 1) / kChanPerCta, groups),
                    dim3(kWarps * 32), smem2, st, false, P);
  if (e != cudaSuccess) return e;
  return launch_kernel("combine", k_combine, dim3(a.T), dim3(256), 0, st, false, a.T, c.hidden, c.n_experts,
                       c.top_k, a.topk_ids, a.topk_w, a.slot_pos, (const float*)a.y_slot,
                       (const float*)(c.shared_inter > 0 ? a.ys : nullptr), a.out);
}

}  // namespace v4moe
