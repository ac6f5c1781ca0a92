// Combine of the routed expert outputs and the shared term for the
// small-batch tensor-core path (8 < T < 512; larger batches fuse it into the
// shared expert's down projection):
//   out[t] = bf16( sum_j w[t, j] * y_slot[slot(t, j)] + ys[t] )   (y_slot bf16, ys fp32)
// summed in slot order j = 0 .. k-1, then the shared term ("Checked in its
// code" rows "Mixture of experts" and "Shared expert"), so the result does not
// depend on timing. Out-of-range expert ids contribute nothing (the router or
// the caller's routing flags them).
#include <cuda_bf16.h>

#include "launch.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

// out[t] = bf16(sum_j w[t,j] * y_slot[slot_pos[t*k+j]] + ys[t]), j in order.
__global__ void __launch_bounds__(256) k_combine(int T, int H, int E, int k, const int32_t* __restrict__ ids,
                                                 const float* __restrict__ w, const int32_t* __restrict__ slot_pos,
                                                 const __nv_bfloat16* __restrict__ y_slot, const float* __restrict__ ys,
                                                 __nv_bfloat16* __restrict__ out) {
  const int t = blockIdx.x;
  for (int m = threadIdx.x * 4; m < H; m += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int e = ids[size_t(t) * k + j];
      if (e < 0 || e >= E) continue;
      const float wj = w[size_t(t) * k + j];
      const uint2 y = *reinterpret_cast<const uint2*>(y_slot + size_t(slot_pos[size_t(t) * k + j]) * H + m);
      acc.x = fmaf(wj, __uint_as_float(y.x << 16), acc.x);
      acc.y = fmaf(wj, __uint_as_float(y.x & 0xFFFF0000u), acc.y);
      acc.z = fmaf(wj, __uint_as_float(y.y << 16), acc.z);
      acc.w = fmaf(wj, __uint_as_float(y.y & 0xFFFF0000u), acc.w);
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
                       c.top_k, a.topk_ids, a.topk_w, a.slot_pos, (const __nv_bfloat16*)a.y_slot,
                       (const float*)(c.shared_inter > 0 ? a.ys : nullptr), a.out);
}

}  // namespace v4moe
