// Internal declarations shared by the libv4moe translation units.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/v4moe.h"

namespace v4moe {

// Status block (first 256 bytes of the workspace): word 0 is the device
// status word.
// Device status word bits.
constexpr uint32_t kStatusBadExpertId = 1u << 0;
constexpr uint32_t kStatusBadTokenId = 1u << 1;
constexpr uint32_t kStatusTimeout = 1u << 2;

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

// Slots per chunk of the multi-CTA permutation.
constexpr int kPermChunk = 2048;

// Host checks shared by every entry point: the config's shape rules, and the
// current device (compute capability 10.0). Device attributes are queried once
// per device and cached (thread-safe); device_sms() is the cached SM count.
bool config_ok(const v4moe_config* c);
int32_t check_device();
int device_sms();

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to
// libcuda), looked up once; null when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// A tiled map of rank 2 or 3 with unit element strides, no
// interleave, L2 promotion of 256 bytes and no fill. dims / box list the
// innermost dimension first; strides[i] is the byte stride of dimension i + 1.
// False when the entry point is missing or the driver rejects the map.
bool encode_tensor_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw);

size_t tc_extra_bytes(const v4moe_config& c, int64_t T);

// Router GEMM: the reduction is split so that about this many CTAs run; the
// workspace holds ksplit partial logit arrays [T, E].
constexpr int kRouteTargetCtas = 148;
int route_ksplit(const v4moe_config& c, int64_t T);

// Shared expert on the token-major f16 GEMM (int8 weights widened to f16 in
// the workspace) from this many tokens on.
constexpr int kShMinTokens = 512;
size_t sh_extra_bytes(const v4moe_config& c, int64_t T);

// Buffers of the decode path (all zero bytes when T is above its limit). ctl
// holds the routing tables.
struct DecodeBuffers {
  size_t ctl = 0, dh = 0, hs = 0;
};
DecodeBuffers dec_buffers(const v4moe_config& c, int64_t T);

// Workspace carve-up for T tokens. All offsets are 256-byte aligned.
struct WsLayout {
  size_t status = 0;        // uint32 status word + spare words (256 B)
  size_t scores = 0;        // router: [ksplit, T, E] fp32 partial logits
  size_t chunk_counts = 0;  // [nchunks, E] int32
  size_t chunk_base = 0;    // [nchunks, E] int32
  size_t h = 0;             // [T*k, I] bf16 routed intermediates (sorted order)
  size_t y_slot = 0;        // [T*k, H] bf16 routed expert outputs (sorted order)
  size_t hs = 0;            // [T, I_s] bf16 shared intermediates
  size_t ys = 0;            // [T, H] fp32 shared expert outputs
  size_t xlog = 0;          // [T, H] f16 activations in the decode layout
  size_t sigma = 0;         // [T] int32 per-token power-of-two exponents
  size_t tc = 0;            // tensor-core path: activations in slot order + tile lists
  size_t sh16 = 0;          // shared expert weights widened to f16 (large batches)
  size_t d_ctl = 0, d_dh = 0, d_hs = 0;  // decode path
  size_t total = 0;
  int nchunks = 0;
};

inline WsLayout ws_layout(const v4moe_config& c, int64_t T) {
  WsLayout L;
  const int64_t S = T * c.top_k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  L.status = take(256);
  L.scores = take(size_t(route_ksplit(c, T)) * T * c.n_experts * 4);
  L.nchunks = int((S + kPermChunk - 1) / kPermChunk);
  if (L.nchunks < 1) L.nchunks = 1;
  L.chunk_counts = take(size_t(L.nchunks) * c.n_experts * 4);
  L.chunk_base = take(size_t(L.nchunks) * c.n_experts * 4);
  L.h = take(size_t(S) * c.inter * 2);
  L.y_slot = take(size_t(S) * c.hidden * 2);
  L.hs = take(size_t(T) * (c.shared_inter > 0 ? c.shared_inter : 0) * 2);
  L.ys = take(size_t(T) * c.hidden * 4);
  L.xlog = take(size_t(T) * c.hidden * 2);
  L.sigma = take(size_t(T) * 4);
  L.tc = take(tc_extra_bytes(c, T));
  L.sh16 = take(sh_extra_bytes(c, T));
  const DecodeBuffers d = dec_buffers(c, T);
  L.d_ctl = take(d.ctl);
  L.d_dh = take(d.dh);
  L.d_hs = take(d.hs);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- launchers
// Each returns cudaGetLastError() of its launches.
// Router (any T): tcgen05 gate GEMM into the partial logits `part`, then the
// per-token selection.
cudaError_t launch_route(const v4moe_config& c, int T, const __nv_bfloat16* x,
                         const __nv_bfloat16* gate, const float* bias, const int32_t* token_ids,
                         const int32_t* tid2eid, int32_t* topk_ids, float* topk_w, float* part,
                         uint32_t* status, cudaStream_t st);

cudaError_t launch_permute(const v4moe_config& c, int T, const int32_t* topk_ids, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos,
                           int32_t* chunk_counts, int32_t* chunk_base, int nchunks,
                           uint32_t* status, cudaStream_t st);

struct ForwardArgs {
  v4moe_config c;
  int T;
  const __nv_bfloat16* x;
  const int32_t* topk_ids;
  const float* topk_w;
  const int32_t* offsets;
  const int32_t* sorted_slot;
  const int32_t* slot_pos;
  v4moe_weights w;
  __nv_bfloat16* out;
  // workspace pieces
  uint32_t* status;
  __nv_bfloat16* h;
  __nv_bfloat16* y_slot;  // routed expert outputs, bf16 (16-bit activations)
  __nv_bfloat16* hs;
  float* ys;
};

cudaError_t launch_combine(const ForwardArgs& a, cudaStream_t st);
// Routed experts on block-scaled tcgen05 MMA (MXFP4 weights as stored, the
// activations as two E4M3 planes with E8M0 scales).
struct MxBuffers {
  uint8_t* xq_hi;  // [S, H] activation planes in slot order
  uint8_t* xq_lo;
  uint8_t* xs_hi;  // [S, H/32] their E8M0 scales
  uint8_t* xs_lo;
  uint8_t* hq_hi;  // [S, I] intermediate planes
  uint8_t* hq_lo;
  uint8_t* hs_hi;  // [S, I/32]
  uint8_t* hs_lo;
};
bool mx_supported(const v4moe_config& c, const v4moe_weights& w);
cudaError_t launch_mx_gather(const ForwardArgs& a, __half* x16, int* sigma, const MxBuffers& m, cudaStream_t st);
// tiles: the tensor-core path's tile list (routed tiles first, shared_tiles
// trailing ones skipped), token tiles of at most bn slots (32, 64 or 128).
// Few tokens per expert: the small token tile leaves room for a deeper ring.
constexpr int kMxSmallTile = 32;
constexpr int kMxSmallAvg = 16;  // slots per expert below which the small tile is used
cudaError_t launch_mx_gemm(const ForwardArgs& a, int w2, const void* tiles, const int* ntiles, int shared_tiles,
                           int bn, const MxBuffers& m, cudaStream_t st);
// Token-major variant (128 slots x 256 weight rows per tile), for experts that
// average at least kMxtMinAvg tokens.
constexpr int kMxtMinAvg = 48;
cudaError_t launch_mxt_gemm(const ForwardArgs& a, int w2, const void* tiles, const int* ntiles, int shared_tiles,
                            const MxBuffers& m, cudaStream_t st);

// Shared expert for at least kShMinTokens tokens: int8 weights widened to f16
// into sh16, then w13 with SwiGLU into hs; w2 with the combine of y_slot fused
// into its epilogue, writing out.
bool sh_supported(const v4moe_config& c, int64_t T);
cudaError_t launch_sh_w13(const ForwardArgs& a, const __half* x16, const int* sigma, char* sh16, cudaStream_t st);
cudaError_t launch_sh_w2_combine(const ForwardArgs& a, char* sh16, cudaStream_t st);

// W8A16 linear in G groups: out[t, g N + n] = bf16(scale[g N + n] *
// sum_k q[g N + n, k] x[t, g K + k]); the int8 weights are widened to bf16 in
// ws (after its 256-byte status block).
size_t linear_w8a16_ws_bytes(int64_t G, int64_t N, int64_t K);
cudaError_t launch_linear_w8a16(int T, int G, int N, int K, const __nv_bfloat16* x, const int8_t* q,
                                const float* scale, __nv_bfloat16* out, char* ws, cudaStream_t st);

// Tensor-core path (tcgen05 grouped GEMMs) for larger token counts.
cudaError_t launch_forward_tc(const ForwardArgs& a, __half* x16, int* sigma, char* extra, char* sh16,
                              cudaStream_t st);

// Decode path: the whole layer (routing included in layer mode) as three
// kernels chained by programmatic dependent launch, for at most
// kDecodeMaxTokens tokens.
constexpr int kDecodeMaxTokens = 8;
struct DecodeArgs {
  v4moe_config c;
  int T;
  int layer_mode;  // 1: route in the kernel; 0: topk ids / weights given
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
  v4moe_weights w;
  __nv_bfloat16* out;
  uint32_t* status;
  uint32_t* ctl;
  __half* dh;
  __half* hs;
};
bool dec_supported(const v4moe_config& c, int T);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// sqrt(softplus(z)) in fp32, softplus in its overflow-free form.
__device__ __forceinline__ float sqrt_softplus_f(float z) {
  const float sp = fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z)));
  return sqrtf(sp);
}

__device__ __forceinline__ float silu_f(float v) { return v / (1.0f + expf(-v)); }

// Clamped SwiGLU: gate clamped from above, up on both sides.
__device__ __forceinline__ float clamped_swiglu_f(float g, float u, float limit) {
  const float gc = fminf(g, limit);
  const float uc = fminf(fmaxf(u, -limit), limit);
  return silu_f(gc) * uc;
}

}  // namespace v4moe
