// Device-side routing and permutation building blocks shared by the router
// kernels and the fused decode preparation kernel.
//  * select_learned / select_hash_warp: one warp selects one token's experts and weights
//    ("Checked in its code" rows "Mixture of experts" and "Auxiliary-loss-free
//    load balancing": top-k of s + bias, weights from the unbiased s, then
//    normalised and multiplied by routed_scaling_factor).
//  * cta_permute: stable counting sort of T*k slots by expert inside one CTA.
#pragma once

#include <cuda_fp16.h>

#include "v4moe_internal.cuh"

namespace v4moe {

// Compare-exchange of (id, value) pairs held identically by every lane.
__device__ __forceinline__ void cswap_pair(int& ia, float& va, int& ib, float& vb) {
  if (ia > ib) {
    const int ti = ia;
    ia = ib;
    ib = ti;
    const float tv = va;
    va = vb;
    vb = tv;
  }
}

// Sort 8 (id, value) pairs by id (odd-even transposition with constant
// indices, so the pairs stay in registers); unused entries carry INT_MAX.
__device__ __forceinline__ void sort8_by_id(int id[8], float v[8]) {
#pragma unroll
  for (int pass = 0; pass < 8; ++pass) {
#pragma unroll
    for (int i = pass & 1; i + 1 < 8; i += 2) cswap_pair(id[i], v[i], id[i + 1], v[i + 1]);
  }
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t float_key(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Learned routing of token t from its E scores s (fp32; SCORE_L2 reads them
// through L2, for scores written by other CTAs of the same kernel): k rounds
// of a warp arg-max over s + bias (largest value, then lowest id), each round
// two warp reductions (largest key, then lowest id holding it); the winner's
// unbiased score comes from its lane. Ids are written in ascending order; w =
// scale * s[id] / sum of the selected s. Every load is issued before the first
// use. NPER bounds the experts per lane (E <= 32 * NPER).
template <bool SCORE_L2, int NPER>
__device__ __forceinline__ void select_learned_n(int t, int E, int k, float routed_scale, const float* s,
                                                 const float* bias, int32_t* __restrict__ topk_ids,
                                                 float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int nper = (E + 31) / 32;
  float sv[NPER], b[NPER];
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    const int ec = (i < nper && e < E) ? e : 0;
    sv[i] = SCORE_L2 ? __ldcg(s + ec) : s[ec];
    b[i] = bias[ec];  // global or shared
  }
  // key 0: not an expert; a NaN sum ranks as -inf
  uint32_t key[NPER];
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    const float v = sv[i] + b[i];
    key[i] = (i < nper && e < E) ? float_key(v != v ? -INFINITY : v) : 0u;
  }
  uint32_t taken = 0;
  int id[8];
  float sel[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    id[r] = 0x7fffffff;
    sel[r] = 0.0f;
    if (r < k) {
      uint32_t lk = 0u;
      int li = 0;
      float ls = 0.0f;
#pragma unroll
      for (int i = 0; i < NPER; ++i)
        if (!((taken >> i) & 1u) && key[i] > lk) {  // strict: lowest id among equal keys
          lk = key[i];
          li = i;
          ls = sv[i];
        }
      const uint32_t mk = __reduce_max_sync(0xffffffffu, lk);
      const uint32_t cand = (lk == mk && lk != 0u) ? uint32_t(lane + 32 * li) : 0xffffffffu;
      const uint32_t wid = __reduce_min_sync(0xffffffffu, cand);
      const float ws = __shfl_sync(0xffffffffu, ls, int(wid & 31u));
      if (lane == int(wid & 31u)) taken |= 1u << (wid >> 5);
      id[r] = int(wid);
      sel[r] = ws;
    }
  }
  sort8_by_id(id, sel);
  float sum = 0.0f;
#pragma unroll
  for (int r = 0; r < 8; ++r) sum += (r < k) ? sel[r] : 0.0f;
  float myv = 0.0f;
  int myid = 0;
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r == lane) {
      myv = sel[r];
      myid = id[r];
    }
  if (lane < k) {
    topk_ids[size_t(t) * k + lane] = myid;
    topk_w[size_t(t) * k + lane] = routed_scale * (myv / sum);
  }
}

template <bool SCORE_L2>
__device__ __forceinline__ void select_learned(int t, int E, int k, float routed_scale, const float* s,
                                               const float* __restrict__ bias, int32_t* __restrict__ topk_ids,
                                               float* __restrict__ topk_w) {
  if (E <= 256)
    select_learned_n<SCORE_L2, 8>(t, E, k, routed_scale, s, bias, topk_ids, topk_w);
  else
    select_learned_n<SCORE_L2, 32>(t, E, k, routed_scale, s, bias, topk_ids, topk_w);
}

// Hash routing of token t (first layers: "select experts from a token-id hash
// table", tid2eid): ids = tid2eid[token_id] in column order, weights from the
// scores s at those ids. Out-of-range token ids / table entries flag the
// status word and give expert 0 with weight 0.
template <bool S_IN_SMEM = false>
__device__ __forceinline__ void select_hash_warp(int t, int E, int k, int vocab, float routed_scale,
                                                 const float* s,
                                                 const int32_t* __restrict__ token_ids,
                                                 const int32_t* __restrict__ tid2eid,
                                                 int32_t* __restrict__ topk_ids, float* __restrict__ topk_w,
                                                 uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int tok = token_ids[t];
  const bool tok_ok = tok >= 0 && tok < vocab;
  int e = 0;
  bool ok = false;
  if (lane < k && tok_ok) {
    e = tid2eid[size_t(tok) * k + lane];
    ok = e >= 0 && e < E;
    if (!ok) e = 0;
  }
  const float v = ok ? (S_IN_SMEM ? s[e] : __ldcg(s + e)) : 0.0f;
  float sum = v;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const unsigned bad = __ballot_sync(0xffffffffu, lane < k && !ok);
  if (bad && lane == 0) atomicOr(status, tok_ok ? kStatusBadExpertId : kStatusBadTokenId);
  if (lane < k) {
    topk_ids[size_t(t) * k + lane] = e;
    topk_w[size_t(t) * k + lane] = (ok && sum > 0.0f) ? routed_scale * (v / sum) : 0.0f;
  }
}

// Walks slots [s0, s1) in order with one warp; cursor[e] (shared) holds the
// next output position of expert e and is advanced. Equal ids within a group
// of 32 are ranked by lane order, so the result is stable.
__device__ __forceinline__ void warp_stable_scatter(const int32_t* ids, int s0, int s1, int E,
                                                    int* cursor, int32_t* __restrict__ sorted_slot,
                                                    int32_t* __restrict__ slot_pos) {
  const int lane = threadIdx.x & 31;
  for (int base = s0; base < s1; base += 32) {
    const int s = base + lane;
    int e = -1;
    if (s < s1) {
      e = ids[s];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (e >= 0) pos = cursor[e] + rank;
    __syncwarp();
    if (e >= 0) {
      const int leader = __ffs(peers) - 1;
      if (lane == leader) cursor[e] += __popc(peers);
      sorted_slot[pos] = s;
      slot_pos[s] = pos;
    }
    __syncwarp();
  }
}

// Whole permutation of S slots inside one CTA (any multiple of 32 threads).
// cnt and cursor are shared arrays of at least E ints.
__device__ __forceinline__ void cta_permute(int S, int E, const int32_t* ids,
                                            int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                            int32_t* __restrict__ sorted_slot, int32_t* __restrict__ slot_pos,
                                            uint32_t* status, int* cnt, int* cursor) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const int e = ids[s];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      bad = true;
  }
  if (bad) atomicOr(status, kStatusBadExpertId);
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int v = e < E ? cnt[e] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (e < E) {
        counts[e] = v;
        offsets[e] = run + incl - v;
        cursor[e] = run + incl - v;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) offsets[E] = run;
    __syncwarp();
    warp_stable_scatter(ids, 0, S, E, cursor, sorted_slot, slot_pos);
  }
  __syncthreads();
}

// Logical K order used by the decode MMA path: inside each 128-element block,
// lane t of a quad owns physical elements [32t, 32t + 32); step s of the block
// uses its elements 4s..4s+3, which land on logical columns 2t, 2t+1, 2t+8,
// 2t+9 of the step's 16. Returns the logical index of physical element j.
__host__ __device__ __forceinline__ int decode_logical_index(int j) {
  const int blk = j >> 7, w = j & 127;
  const int t = w >> 5, q = w & 31;
  const int s = q >> 2, c = q & 3;
  return blk * 128 + s * 16 + (c >> 1) * 8 + 2 * t + (c & 1);
}

// One warp converts a bf16 row of H elements into the decode layout: f16 in
// logical order, scaled by 2^sigma so that the row maximum lies in
// [2^14, 2^15) (exact for every element within 2^-29 of the maximum).
__device__ __forceinline__ void warp_row_to_decode_layout(const __nv_bfloat16* __restrict__ xrow, int H,
                                                          __half* __restrict__ dst, int* sigma_out) {
  const int lane = threadIdx.x & 31;
  const uint4* s4 = reinterpret_cast<const uint4*>(xrow);
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
  if (mx != 0) sg = ef == 0 ? 120 : 141 - ef;  // 14 - floor(log2(max))
  sg = max(-120, min(120, sg));
  if (lane == 0) *sigma_out = sg;
  const float mul = __int_as_float((sg + 127) << 23);
  uint32_t* d32 = reinterpret_cast<uint32_t*>(dst);
#pragma unroll 4
  for (int p = lane; p < H / 8; p += 32) {
    const uint4 v = __ldg(s4 + p);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hv = __floats2half2_rn(__uint_as_float(in[i] << 16) * mul,
                                           __uint_as_float(in[i] & 0xFFFF0000u) * mul);
      d32[decode_logical_index(8 * p + 2 * i) >> 1] = *reinterpret_cast<const uint32_t*>(&hv);
    }
  }
}

}  // namespace v4moe
