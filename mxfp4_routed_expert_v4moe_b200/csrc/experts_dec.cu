// Decode-sized batches (at most 8 tokens): the layer as three kernels chained
// by programmatic dependent launch, streaming every weight byte once.
//
// What it computes ("Checked in its code" rows "Mixture of experts",
// "Auxiliary-loss-free load balancing", "SwiGLU feed-forward", "Shared
// expert"; "config.json" experts_w4a16 / linears_w8a16):
//   layer mode: s[t, e] = sqrt(softplus(gate[e] . x_t)), top-k of s + bias (or
//   the token-id hash table), w = scale * s / sum; forward mode takes ids and
//   weights from the caller. Then, for the shared expert and every routed
//   expert the batch hits,
//     h = silu(min(g, L)) * clamp(u, -L, L),   [g; u] = W13 x_t,
//     out_t = W2_shared hs_t + sum over the token's experts of w * W2_e h.
//
// Kernels:
//  * k_dec_route: one thread-block cluster; each warp scores experts into the
//    leader CTA's shared memory, and after the cluster barrier the leader
//    selects each token's experts and publishes the batch's routing tables
//    (distinct experts in ascending id, token masks, weights), the routing
//    outputs and the permutation.
//  * k_dec_w13: one CTA per SM, two groups of eight warps. Work items are w13
//    slabs (8 channels of a routed expert: 8 gate rows and the 8 matching up
//    rows; or 4 + 4 int8 rows of the shared expert), numbered shared first,
//    then routed expert by expert; CTA b takes a contiguous share of each as
//    its ring positions 0, 1, ..., and group q the positions q, q + 2, ....
//    A CTA reads x, its row scales and the routing tables (in forward mode it
//    builds the tables from the caller's routing) before its first copy, and
//    once its last slab is on its way asks L2 for its share of the routed w2
//    rows. Warp i of a group owns the 128-wide K blocks i, i + 8, ... of a
//    slab, multiplies them by the activations with mma.sync m16n8k16 (f16
//    operands, fp32 accumulation, the tokens as the 8 columns) and posts its
//    partial tile to shared memory; the last warp to post sums the partials
//    in warp order, refills the stage and stages h as f16 (routed: w * h) in
//    shared memory; the CTA writes its h rows once its slabs are done.
//  * k_dec_w2: two groups of eight warps, warp i of a group owning K blocks
//    i, i + 8. CTA b owns a run of (at most two) 16-row output blocks; its
//    ring positions are the blocks' (expert, block) items, the shared expert
//    first, then the routed experts in ascending id, and group q takes the
//    positions q, q + 2, ...; a stage holds the expert's 16 weight rows and
//    the intermediates of its tokens. Each warp sums its items per block in
//    registers; at the end the sixteen warps' sums are added in warp order and
//    written once as bf16, so the result does not depend on timing.
//
// The intermediates are stored as f16 scaled by a fixed power of two chosen
// from the clamp limit: |h| <= L * L * routed_scale, so h * 2^tau stays below
// the f16 maximum for every input while small values keep that many more
// binades; the down projection divides it out.
//
// Operands are exact: E2M1 pairs via cvt.rn.f16x2.e2m1x2, int8 via a
// magic-number conversion. Each 32-wide scale group is its own pair of MMAs
// started from zero, and its E8M0 scale multiplies that result in fp32.
// Activations are f16, scaled per token by a power of two that puts the row
// maximum in [2^14, 2^15).
//
// Weight slabs arrive by TMA as swizzled boxes (a few copies per slab, and
// the eight rows of every fragment load in different banks). A stage's
// consecutive ring positions go to different consumers, so besides its
// mbarrier each stage carries a tag naming the position whose copies were
// issued; a consumer waits for the tag before it tests the barrier's parity.
//
// No CTA waits on another CTA: data crosses kernels only at the programmatic
// launch boundaries (griddepcontrol.wait), which also order memory. Every
// wait is bounded and flags the status word.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>

#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kGW = 8;             // warps per consumer group (w13 kernel)
constexpr int kThreads = 16 * 32;  // both slab kernels
constexpr int kStages13 = 5;
constexpr int kMaxStages2 = 6;
constexpr int kNJ = 4;             // K blocks per warp held in registers (K <= 4096)
constexpr int kMaxHit = 64;        // distinct routed experts of a batch (T * k <= 64)
constexpr int kShRows = 64;        // shared-expert rows per CTA with preloaded scales
constexpr uint32_t kBarTries = 1u << 20;

// Control block words (workspace): the routing tables, rewritten by every
// call for the w2 kernel.
enum Ctl : int {
  cNh = 0,
  cHit = 32,          // [kMaxHit] expert id per list index
  cMask = cHit + 64,  // [kMaxHit] bit per token routed to the expert
  cW = cMask + 64,    // [kMaxHit][8] float weight per (expert, token)
  cWords = cW + 64 * 8,
};

struct DecParams {
  int T, H, I, Is, E, k, vocab;
  float limit, routed_scale;
  float tau_r, tau_s;  // the intermediates are stored as f16(h * tau): routed, shared
  int layer_mode;
  int stage_bytes;
  int nstages;  // w2 ring depth
  int w2_per;   // 16-row output blocks per w2 CTA
  int hrs, hss;  // w13: per-token row capacity of the staged routed / shared intermediates
  const __nv_bfloat16* x;
  const __nv_bfloat16* gate;
  const float* bias;
  const int32_t* token_ids;
  const int32_t* tid2eid;
  int32_t* topk_ids;  // layer mode: written; forward mode: read
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_slot;
  int32_t* slot_pos;
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  const int8_t* sh13;
  const float* sh13_scale;
  const int8_t* sh2;
  const float* sh2_scale;
  __half* dh;  // [kMaxHit, T, I] weighted routed intermediates
  __half* hs;  // [T, Is] shared intermediates
  uint32_t* ctl;
  uint32_t* status;
  __nv_bfloat16* out;
};

// Tensor maps of a slab kernel's weights (u8 views, built on the host):
// codes {128, rows, K / 256 chunks} with box {128, 8 or 16, K / 256}, scales
// {K / 32, rows} with box {K / 32, 8 or 16}, shared-expert int8 rows {128,
// rows, K / 128} with box {128, 4 or 16, K / 128}.
struct DecMaps {
  CUtensorMap codes, scales, shared;
};

// Routing tables as the slab kernels keep them in shared memory.
struct Tables {
  int nh;
  int hit[kMaxHit];
  uint32_t mask[kMaxHit];
  float w[kMaxHit * 8];
};

__device__ __forceinline__ float pow2f(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((e + 127) << 23);
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const DecParams& P) {
  if (mbar_wait_bounded(bar, parity, kBarTries)) return true;
  atomicOr(P.status, kStatusTimeout);
  return false;
}

// Waits until ring stage `bar` / `tag` holds position pos of a ring of ns
// stages. Consecutive positions of a stage (pos - ns, pos) go to different
// consumers, so a consumer can reach pos while the stage still holds pos - ns;
// the barrier's parity alone would then take the older phase's completion for
// this one. The tag names the last position whose copies were issued: it is
// written after pos - ns was consumed and before pos's copies, so once it
// reads pos the barrier's current phase is pos's.
__device__ __forceinline__ bool wait_stage(uint64_t* bar, const int* tag, int pos, int ns, const DecParams& P) {
  uint32_t i = 0;
  while (*reinterpret_cast<const volatile int*>(tag) != pos && ++i < kBarTries) __nanosleep(20);
  if (i >= kBarTries) {
    atomicOr(P.status, kStatusTimeout);
    return false;
  }
  return wait_bar(bar, uint32_t(pos / ns) & 1u, P);
}

// 14 - floor(log2 m) for the largest bf16 magnitude bits m of a row (0 for an
// all-zero row), clamped to [-120, 120]: 2^sigma * max lies in [2^14, 2^15).
__device__ __forceinline__ int sigma_of(uint32_t mx) {
  if (mx == 0) return 0;
  const int ef = int(mx >> 7);
  const int sg = ef == 0 ? 120 : 141 - ef;
  return max(-120, min(120, sg));
}

__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t m, uint32_t w) {
  return max(m, max(w & 0x7FFFu, (w >> 16) & 0x7FFFu));
}

// Whole CTA; the caller synchronises afterwards.
__device__ __forceinline__ void read_tables(Tables& tb, const DecParams& P) {
  const int nh = min(max(int(__ldcg(P.ctl + cNh)), 0), kMaxHit);  // bounded whatever the word holds
  for (int i = threadIdx.x; i < nh; i += blockDim.x) {
    tb.hit[i] = int(__ldcg(P.ctl + cHit + i));
    tb.mask[i] = __ldcg(P.ctl + cMask + i);
  }
  for (int i = threadIdx.x; i < nh * 8; i += blockDim.x) tb.w[i] = __ldcg(reinterpret_cast<const float*>(P.ctl + cW) + i);
  if (threadIdx.x == 0) tb.nh = nh;
}

// ---------------------------------------------------------------- slab products

// Slab layout in a stage. Weight rows arrive by TMA as boxes {128 bytes,
// rows, chunks}: chunk c (bytes 128 c .. 128 c + 127) of every row of the box,
// then chunk c + 1, ..., so row r's chunk c is line c * rows + r of the box.
// The 128-byte swizzle permutes the eight 16-byte units of each line by the
// line index mod 8; the eight rows a fragment load touches are eight
// consecutive lines, so their units fall in eight different bank groups. Row
// scales arrive as boxes {S bytes, rows} (S = K / 32) with the swizzle of span
// S (none at 16 bytes). Every box starts at a multiple of 1024 bytes, the
// period of the swizzle.
__device__ __forceinline__ int swz(int o, int mask) { return o ^ (((o >> 7) & mask) << 4); }

// Swizzle mask of a scale box with S-byte rows (S a power of two, 16 .. 128).
__host__ __device__ constexpr int scale_mask(int S) { return S >= 128 ? 7 : S / 16 - 1; }

__host__ __device__ constexpr int align1k(int b) { return (b + 1023) / 1024 * 1024; }

// K order of the MMA steps. In a 128-wide K block, 32-wide group q (one E8M0
// scale per weight row) feeds two m16n8k16 steps h = 0, 1; lane quad member
// t owns the group's elements 8 t .. 8 t + 7 and gives elements 8 t + 4 h +
// {0, 1, 2, 3} to the step's logical columns 2t, 2t + 1, 2t + 8, 2t + 9 (A
// and B alike). The B fragment of a K block is therefore, per q, the 8
// activations 32 q + 8 t .. + 7 of token g: B[4 q .. 4 q + 3].

// MXFP4 m16 tile: tile row g is row ra of code box ca, tile row g + 8 is row
// rb of code box cb (both boxes of nrows rows); their E8M0 scales are rows ra
// / rb of scale boxes sa / sb (S bytes per row). The warp's K blocks kb = wi
// + KS j (j < NJ, kb < nkb) multiply B[j]. Each group's two MMAs start from
// zero and the group's scales multiply the result into acc (fp32), so the
// E2M1 operands need no scaling.
template <int NJ, int KS>
__device__ __forceinline__ void tile_mx(const char* ca, int ra, const char* cb, int rb, int nrows, const char* sa,
                                        const char* sb, int S, int wi, int nkb, const uint32_t (&B)[NJ][16],
                                        float (&acc)[4]) {
  const int t = threadIdx.x & 3;
  const int sm = scale_mask(S);
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int kb = wi + KS * j;
    if (kb < nkb) {
      // the block's 4 group exponents of each row
      const uint32_t ea = lds32(sa + swz(ra * S + 4 * kb, sm));
      const uint32_t eb = lds32(sb + swz(rb * S + 4 * kb, sm));
      const int la = (kb >> 1) * nrows + ra, lb = (kb >> 1) * nrows + rb;  // lines of the rows' chunk
      const int u0 = (kb & 1) << 2;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t wa = lds32(ca + la * 128 + (((u0 + q) ^ (la & 7)) << 4) + 4 * t);
        const uint32_t wb = lds32(cb + lb * 128 + (((u0 + q) ^ (lb & 7)) << 4) + 4 * t);
        uint32_t xa[4], xb[4];
        e2m1x8_to_f16x2(wa, xa);
        e2m1x8_to_f16x2(wb, xb);
        const uint32_t A0[4] = {xa[0], xb[0], xa[1], xb[1]};
        const uint32_t A1[4] = {xa[2], xb[2], xa[3], xb[3]};
        float d[4];
        mma_16816_f16_zero(d, A0, B[j][4 * q], B[j][4 * q + 1]);
        mma_16816_f16(d, A1, B[j][4 * q + 2], B[j][4 * q + 3]);
        // E8M0 e is 2^(e - 127): the float with exponent field e
        const float fa = __uint_as_float(((ea >> (8 * q)) & 0xFFu) << 23);
        const float fb = __uint_as_float(((eb >> (8 * q)) & 0xFFu) << 23);
        acc[0] = fmaf(d[0], fa, acc[0]);
        acc[1] = fmaf(d[1], fa, acc[1]);
        acc[2] = fmaf(d[2], fb, acc[2]);
        acc[3] = fmaf(d[3], fb, acc[3]);
      }
    }
  }
}

// int8 m16 tile: tile rows g / g + 8 are row ra of box ca / row rb of box cb
// (chunked boxes of nrows rows), zero rows where `valid` is false; the warp's
// K blocks kb = wi + KS j < nkb. Accumulates in ae (steps h = 0) and ao (h = 1).
template <int NJ, int KS>
__device__ __forceinline__ void tile_s8(const char* ca, int ra, const char* cb, int rb, int nrows, bool valid, int wi,
                                        int nkb, const uint32_t (&B)[NJ][16], float (&ae)[4], float (&ao)[4]) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int kb = wi + KS * j;
    if (kb < nkb) {
      const int la = kb * nrows + ra, lb = kb * nrows + rb;  // a K block is one chunk
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint2 qa = make_uint2(0u, 0u), qb = qa;
        if (valid) {
          const int u = 2 * q + (t >> 1), w = 8 * (t & 1);
          qa = lds64(ca + la * 128 + ((u ^ (la & 7)) << 4) + w);
          qb = lds64(cb + lb * 128 + ((u ^ (lb & 7)) << 4) + w);
        }
        uint32_t A[4];
        s8x4_to_f16x2(qa.x, A[0], A[2]);
        s8x4_to_f16x2(qb.x, A[1], A[3]);
        mma_16816_f16(ae, A, B[j][4 * q], B[j][4 * q + 1]);
        s8x4_to_f16x2(qa.y, A[0], A[2]);
        s8x4_to_f16x2(qb.y, A[1], A[3]);
        mma_16816_f16(ao, A, B[j][4 * q + 2], B[j][4 * q + 3]);
      }
    }
  }
}

// B fragments of K block kb for token row `row` (f16 elements, K block at kb
// * 128): per group q the 8 activations 32 q + 8 t .. + 7.
__device__ __forceinline__ void load_b_smem(const char* row, int kb, uint32_t (&B)[16]) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = lds128(row + (kb * 128 + 32 * q + 8 * t) * 2);
    B[4 * q] = v.x;
    B[4 * q + 1] = v.y;
    B[4 * q + 2] = v.z;
    B[4 * q + 3] = v.w;
  }
}

// ---------------------------------------------------------------- routing

// Selection and routing tables, built in shared memory by every w13 CTA.
struct RouteSmem {
  uint32_t bits[32];
  int rank_base[32];
  int cnt[kMaxHit];
  int cum[kMaxHit + 1];
  int ids[64];
  float wts[64];
  int32_t sel_ids[64];  // the selection's output
  float sel_w[64];
};

// The batch's routed experts in ascending id, per (expert, token) weights and
// token masks, from topk ids / weights (global or shared memory), into tb;
// one warp. Out-of-range ids are skipped and, unless `quiet`, flagged.
__device__ __forceinline__ void route_tables(RouteSmem& S, Tables& tb, const DecParams& P, const int32_t* tids,
                                             const float* tw, bool quiet) {
  const int lane = threadIdx.x & 31;
  const int Sn = P.T * P.k;
  S.bits[lane] = 0u;
  __syncwarp();
  bool bad = false;
  for (int s = lane; s < 64; s += 32) {
    int e = -1;
    float w = 0.f;
    if (s < Sn) {
      e = tids[s];
      w = tw[s];
      if (e < 0 || e >= P.E) {
        bad = true;
        e = -1;
      }
    }
    S.ids[s] = e;
    S.wts[s] = w;
    if (e >= 0) atomicOr(&S.bits[e >> 5], 1u << (e & 31));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && !quiet) atomicOr(P.status, kStatusBadExpertId);
  __syncwarp();
  const uint32_t word = S.bits[lane];
  const int c = __popc(word);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  S.rank_base[lane] = incl - c;
  const int nh = __shfl_sync(0xffffffffu, incl, 31);
  for (int i = lane; i < kMaxHit * 8; i += 32) tb.w[i] = 0.f;
  for (int i = lane; i < kMaxHit; i += 32) {
    tb.mask[i] = 0u;
    S.cnt[i] = 0;
  }
  __syncwarp();
  for (int s = lane; s < Sn; s += 32) {
    const int e = S.ids[s];
    if (e >= 0) {
      const int r = S.rank_base[e >> 5] + __popc(S.bits[e >> 5] & ((1u << (e & 31)) - 1u));
      const int tok = s / P.k;
      tb.hit[r] = e;
      atomicAdd(&tb.w[r * 8 + tok], S.wts[s]);
      atomicOr(&tb.mask[r], 1u << tok);
      atomicAdd(&S.cnt[r], 1);
    }
  }
  if (lane == 0) tb.nh = nh;
  __syncwarp();
}

// The tables, for the w2 kernel (one warp).
__device__ __forceinline__ void publish_tables(const Tables& tb, const DecParams& P) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < tb.nh; i += 32) {
    P.ctl[cHit + i] = uint32_t(tb.hit[i]);
    P.ctl[cMask + i] = tb.mask[i];
  }
  for (int i = lane; i < tb.nh * 8; i += 32) reinterpret_cast<float*>(P.ctl + cW)[i] = tb.w[i];
  if (lane == 0) P.ctl[cNh] = uint32_t(tb.nh);
}

// Stable counting sort of the batch's slots by expert (layer-mode outputs),
// from the state route_tables left in shared memory; one warp.
__device__ __forceinline__ void write_permutation(RouteSmem& S, const DecParams& P, int nh) {
  const int lane = threadIdx.x & 31;
  const int Sn = P.T * P.k;
  const int c0 = 2 * lane < nh ? S.cnt[2 * lane] : 0;
  const int c1 = 2 * lane + 1 < nh ? S.cnt[2 * lane + 1] : 0;
  int incl = c0 + c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  const int excl = incl - c0 - c1;
  S.cum[2 * lane] = excl;
  S.cum[2 * lane + 1] = excl + c0;
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (lane == 0) S.cum[kMaxHit] = total;
  __syncwarp();
  for (int e = lane; e < P.E; e += 32) {
    const uint32_t word = S.bits[e >> 5];
    const int r = S.rank_base[e >> 5] + __popc(word & ((1u << (e & 31)) - 1u));
    const bool hit = (word >> (e & 31)) & 1u;
    P.counts[e] = hit ? S.cnt[r] : 0;
    P.offsets[e] = r < nh ? S.cum[r] : total;
  }
  if (lane == 0) P.offsets[P.E] = total;
  for (int s = lane; s < Sn; s += 32) {
    const int e = S.ids[s];
    if (e < 0) continue;
    const int r = S.rank_base[e >> 5] + __popc(S.bits[e >> 5] & ((1u << (e & 31)) - 1u));
    int before = 0;
    for (int s2 = 0; s2 < s; ++s2) before += S.ids[s2] == e;
    const int pos = S.cum[r] + before;
    P.sorted_slot[pos] = s;
    P.slot_pos[s] = pos;
  }
}

constexpr int kRouteWarps = 16;
constexpr int kRouteMaxCluster = 16;

// Learned routing of token t by one warp from E <= 32 NPER scores s and bias b
// in shared memory: k rounds of a warp arg-max over s + b (larger key, then
// lower id), then the k winners ordered by id and w = scale * s / (their sum
// in that order) -- the same selection, ties and rounding as
// select_learned_n, written as loops: the router runs it once per call with
// its instructions not yet in any cache, so its length is its latency.
template <int NPER>
__device__ __noinline__ void select_compact(int t, int E, int k, float scale, const float* s, const float* b,
                                            int32_t* ids, float* w) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NPER];  // 0: not an expert, or already taken
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    float v = 0.f;
    if (e < E) v = s[e] + b[e];
    key[i] = e < E ? float_key(v != v ? -INFINITY : v) : 0u;
  }
  int myid = 0x7fffffff;  // lane r < k: the winner of round r
  float myv = 0.f;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    uint32_t lk = 0u;
    int li = 0;
#pragma unroll
    for (int i = 0; i < NPER; ++i)
      if (key[i] > lk) {  // strict: the lowest id among equal keys
        lk = key[i];
        li = i;
      }
    const uint32_t mk = __reduce_max_sync(0xffffffffu, lk);
    const uint32_t cand = (lk == mk && lk != 0u) ? uint32_t(lane + 32 * li) : 0xffffffffu;
    const uint32_t wid = __reduce_min_sync(0xffffffffu, cand);
    if (lane == int(wid & 31u))
#pragma unroll
      for (int i = 0; i < NPER; ++i)
        if (i == int(wid >> 5)) key[i] = 0u;
    if (lane == r) {
      myid = int(wid);
      myv = wid < uint32_t(E) ? s[wid] : 0.f;
    }
  }
  int rank = 0;  // position of this lane's winner in ascending id order
#pragma unroll 1
  for (int j = 0; j < k; ++j) rank += __shfl_sync(0xffffffffu, myid, j) < myid;
  float sum = 0.f;
#pragma unroll 1
  for (int p = 0; p < k; ++p) {
    const unsigned m = __ballot_sync(0xffffffffu, lane < k && rank == p);
    sum += __shfl_sync(0xffffffffu, myv, __ffs(m) - 1);
  }
  if (lane < k) {
    ids[size_t(t) * k + rank] = myid;
    w[size_t(t) * k + rank] = scale * (myv / sum);
  }
}

// What the router's leader CTA keeps in shared memory besides the scores.
struct RouteTail {
  RouteSmem rt;
  Tables tb;
};
constexpr size_t kRouteTail = (sizeof(RouteTail) + 15) / 16 * 16;

// Router: one thread-block cluster of CL CTAs. Warp w of CTA r scores experts
// e = r * kRouteWarps + w, + CL * kRouteWarps, ... (one warp per expert, the
// x rows staged in shared memory) and stores s[t, e] into the leader CTA's
// shared memory; after the cluster barrier the leader (rank 0) selects each
// token's experts (bias prefetched into its shared memory), builds the
// batch's routing tables (distinct experts in ascending id, token masks,
// weights) and writes them for the slab kernels, with the routing outputs and
// the permutation. Shared memory: tail, scores [T][E], bias [E], x [T][H].
__global__ void __launch_bounds__(kRouteWarps * 32) k_dec_route(DecParams P) {
  extern __shared__ __align__(16) char rsm[];
  RouteTail& R = *reinterpret_cast<RouteTail*>(rsm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = P.H, T = P.T, E = P.E;
  float* sc = reinterpret_cast<float*>(rsm + kRouteTail);
  float* sb = sc + size_t(T) * E;
  uint4* xs = reinterpret_cast<uint4*>(rsm + kRouteTail + ((size_t(T) * E + E) * 4 + 15) / 16 * 16);
  const uint32_t rank = cluster_ctarank();
  const int CL = int(gridDim.x);
  // The w13 kernel may start now: before it waits for this grid it reads only
  // the activations and weights and issues its shared-expert copies.
  pdl_launch_dependents();
  const int np = H / 8 / 32;
  int e = int(rank) * kRouteWarps + warp;
  // the first gate row in flight at once (H <= 4096: up to 16 pieces per lane)
  uint4 gv[16];
  {
    const uint4* grow = reinterpret_cast<const uint4*>(P.gate + size_t(e < E ? e : 0) * H);
#pragma unroll
    for (int i = 0; i < 16; ++i) gv[i] = i < np ? __ldg(grow + lane + 32 * i) : make_uint4(0u, 0u, 0u, 0u);
  }
  for (int i = threadIdx.x; i < T * H / 8; i += blockDim.x) xs[i] = __ldg(reinterpret_cast<const uint4*>(P.x) + i);
  if (rank == 0 && P.bias)
    for (int i = threadIdx.x; i < E; i += blockDim.x) sb[i] = __ldg(P.bias + i);
  __syncthreads();
  for (; e < E; e += CL * kRouteWarps) {
    if (e >= int(rank) * kRouteWarps + kRouteWarps) {  // a further row
      const uint4* grow = reinterpret_cast<const uint4*>(P.gate + size_t(e) * H);
#pragma unroll
      for (int i = 0; i < 16; ++i) gv[i] = i < np ? __ldg(grow + lane + 32 * i) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int t = 0; t < T; ++t) {
      const uint4* xrow = xs + size_t(t) * (H / 8);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < np) {
          const uint4 xv = xrow[lane + 32 * i];
          acc = fmaf(bf16_lo(gv[i].x), bf16_lo(xv.x), acc);
          acc = fmaf(bf16_hi(gv[i].x), bf16_hi(xv.x), acc);
          acc = fmaf(bf16_lo(gv[i].y), bf16_lo(xv.y), acc);
          acc = fmaf(bf16_hi(gv[i].y), bf16_hi(xv.y), acc);
          acc = fmaf(bf16_lo(gv[i].z), bf16_lo(xv.z), acc);
          acc = fmaf(bf16_hi(gv[i].z), bf16_hi(xv.z), acc);
          acc = fmaf(bf16_lo(gv[i].w), bf16_lo(xv.w), acc);
          acc = fmaf(bf16_hi(gv[i].w), bf16_hi(xv.w), acc);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) st_cluster_f32(map_to_rank(sc + size_t(t) * E + e, 0), sqrt_softplus_f(acc));
    }
  }
  cluster_sync_all();  // every score is in the leader's shared memory
  if (rank != 0) return;
  // ---- the leader routes the batch
  if (warp < T) {
    const float* st = sc + size_t(warp) * E;
    if (P.token_ids)  // scores in shared memory
      select_hash_warp<true>(warp, E, P.k, P.vocab, P.routed_scale, st, P.token_ids, P.tid2eid, R.rt.sel_ids,
                             R.rt.sel_w, P.status);
    else if (E <= 256)
      select_compact<8>(warp, E, P.k, P.routed_scale, st, sb, R.rt.sel_ids, R.rt.sel_w);
    else
      select_compact<32>(warp, E, P.k, P.routed_scale, st, sb, R.rt.sel_ids, R.rt.sel_w);
  }
  __syncthreads();
  if (warp == 0) route_tables(R.rt, R.tb, P, R.rt.sel_ids, R.rt.sel_w, true);
  __syncthreads();
  if (warp == 0) publish_tables(R.tb, P);
  if (warp == 1)
    for (int i = lane; i < T * P.k; i += 32) {
      P.topk_ids[i] = R.rt.sel_ids[i];
      P.topk_w[i] = R.rt.sel_w[i];
    }
  if (warp == 2) write_permutation(R.rt, P, R.tb.nh);
}

// ---------------------------------------------------------------- w13 kernel

struct W13Smem {
  uint64_t full[kStages13];
  int redcnt[kStages13];
  int lastfill[kStages13];
  int sigma[2][8];  // per consumer group
  uint32_t xmax[2][kGW][8];
  float sh_scale[2][kShRows];  // gate / up row scales of this CTA's shared slabs
  Tables tb;
  RouteSmem rt;
};

constexpr size_t kHead13 = (sizeof(W13Smem) + 127) / 128 * 128;
constexpr size_t kPart13 = size_t(kStages13) * kGW * 32 * 16;  // float4 per lane and warp

enum Kind : int { kEnd = 0, kS13 = 1, kR13 = 2 };
struct Item {
  int kind, li, row0, e;
};

// Item number -> slab: shared w13 slabs (4 gate + 4 up int8 rows) first, then
// routed w13 slabs (8 + 8 MXFP4 rows), expert by expert.
__device__ __forceinline__ Item w13_item(const DecParams& P, const Tables& tb, int it) {
  Item m = {kEnd, 0, 0, 0};
  const int n_s = P.Is > 0 ? P.Is / 4 : 0;
  if (it < n_s) {
    m.kind = kS13;
    m.row0 = it * 4;
  } else {
    const int r = it - n_s, i8 = P.I / 8;
    if (r < tb.nh * i8) {
      m.kind = kR13;
      m.li = r / i8;
      m.row0 = (r % i8) * 8;
      m.e = tb.hit[m.li];
    }
  }
  return m;
}

// Copies slab m into stage s (lane 0 of the calling warp issues and arms):
// routed, the gate and up code boxes (8 rows each) and their scale boxes;
// shared, the 4 gate and 4 up int8 rows as two boxes.
__device__ __forceinline__ void fill13(const DecParams& P, const DecMaps& M, W13Smem& S, char* dst, int s,
                                       const Item& m, int pos) {
  const int H = P.H;
  if ((threadIdx.x & 31) == 0) {
    S.lastfill[s] = pos;
    if (m.kind == kS13) {
      mbar_arrive_expect_tx(&S.full[s], uint32_t(8 * H));
      tma_load_3d(dst, &M.shared, 0, m.row0, 0, &S.full[s]);
      tma_load_3d(dst + 4 * H, &M.shared, 0, P.Is + m.row0, 0, &S.full[s]);
    } else {
      const int rg = m.e * 2 * P.I + m.row0, ru = rg + P.I;
      const int sc = 8 * H, sbox = align1k(8 * (H / 32));
      mbar_arrive_expect_tx(&S.full[s], uint32_t(8 * H + 16 * (H / 32)));
      tma_load_3d(dst, &M.codes, 0, rg, 0, &S.full[s]);
      tma_load_3d(dst + 4 * H, &M.codes, 0, ru, 0, &S.full[s]);
      tma_load_2d(dst + sc, &M.scales, 0, rg, &S.full[s]);
      tma_load_2d(dst + sc + sbox, &M.scales, 0, ru, &S.full[s]);
    }
  }
  __syncwarp();
}

// CTA b's share of the w13 slabs: shared slabs [s0, s1) and routed slabs
// [r0, r1) (routed slab r is item n_s + r), contiguous so that each expert's
// rows form one range per CTA. Ring position p is the p-th of these.
struct Chunk {
  int s0, s1, r0, r1;
  __device__ int size() const { return (s1 - s0) + (r1 - r0); }
  __device__ int item(int p, int n_s) const { return p < s1 - s0 ? s0 + p : n_s + r0 + (p - (s1 - s0)); }
};
__device__ __forceinline__ Chunk w13_chunk(const DecParams& P, int nh, int b, int G) {
  Chunk c;
  const int n_s = P.Is > 0 ? P.Is / 4 : 0, n_r = nh * (P.I / 8);
  const int per_s = (n_s + G - 1) / G, per_r = (n_r + G - 1) / G;
  c.s0 = min(n_s, b * per_s);
  c.s1 = min(n_s, c.s0 + per_s);
  c.r0 = min(n_r, b * per_r);
  c.r1 = min(n_r, c.r0 + per_r);
  return c;
}

// The w2 rows of the 16-row output blocks that CTA b of the w2 kernel owns
// (blocks [b w2_per, (b + 1) w2_per)): the shared expert's, or every routed
// expert's (one lane).
__device__ __forceinline__ void prefetch_w2_share(const DecParams& P, const Tables& tb, int b, bool routed) {
  const int nrb = P.H / 16;
  const int rb0 = min(nrb, b * P.w2_per), rb1 = min(nrb, rb0 + P.w2_per);
  if (rb1 <= rb0) return;
  const size_t rows = size_t(16) * (rb1 - rb0);
  if (!routed) {
    if (P.Is > 0) prefetch_l2_range(reinterpret_cast<const char*>(P.sh2) + size_t(16 * rb0) * P.Is, rows * P.Is);
    return;
  }
  for (int li = 0; li < tb.nh; ++li) {
    const size_t r0 = size_t(tb.hit[li]) * P.H + size_t(16) * rb0;
    prefetch_l2_range(P.w2_codes + r0 * (P.I / 2), rows * (P.I / 2));
    prefetch_l2_range(P.w2_scales + r0 * (P.I / 32), rows * (P.I / 32));
  }
}

__global__ void __launch_bounds__(kThreads, 1) k_dec_w13(DecParams P, const __grid_constant__ DecMaps M) {
  extern __shared__ __align__(128) char smem[];
  W13Smem& S = *reinterpret_cast<W13Smem*>(smem);
  // Test hook (word 1 of the status block, zero in normal use): a wait on a
  // barrier that nothing arrives at, bounded by that many polls; it gives up,
  // flags the timeout and the CTA returns before issuing any copy.
  if (const uint32_t arm = __ldcg(P.status + 1)) {
    if (threadIdx.x == 0) {
      mbar_init(&S.full[0], 1);
      fence_mbar_init();
      if (!mbar_wait_bounded(&S.full[0], 0u, arm)) atomicOr(P.status, kStatusTimeout);
    }
    return;
  }
  // stages at the next multiple of 1024 bytes (the swizzle's period)
  char* stages = smem + ((smem_u32(smem) + uint32_t(kHead13) + 1023u) & ~1023u) - smem_u32(smem);
  float4* parts = reinterpret_cast<float4*>(stages + size_t(kStages13) * P.stage_bytes);
  // This CTA's intermediates, written to global memory once its slabs are
  // done (a global store in the slab loop would wait behind the SM's copies
  // in flight, and so would the fences after it): routed [T][hrs], shared
  // [T][hss], rows in the order of the CTA's slabs.
  __half* hst_r = reinterpret_cast<__half*>(reinterpret_cast<char*>(parts) + kPart13);
  __half* hst_s = hst_r + size_t(P.T) * P.hrs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = P.T, H = P.H;
  const int G = int(gridDim.x), b = int(blockIdx.x);
  const int n_s = P.Is > 0 ? P.Is / 4 : 0;
  const int q = warp / kGW, wi = warp % kGW;
  const int g = lane >> 2, t = lane & 3;
  const int nkbH = H / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages13; ++s) {
      mbar_init(&S.full[s], 1);
      S.redcnt[s] = 0;
      S.lastfill[s] = -1;
    }
    S.tb.nh = 0;
    fence_mbar_init();
  }
  // The w2 kernel may launch now (its CTAs start as these leave their SMs).
  pdl_launch_dependents();

  // Everything this CTA reads from global memory outside the ring is read
  // before its first copy goes out: on this GPU a load, like an instruction
  // fetch, waits behind the SM's copies in flight. First what does not
  // depend on the previous grid: this warp's x slices (token g, K blocks wi
  // + 8 j; per 32-wide group p the activations kb * 128 + 32 p + 8 t .. + 7,
  // the MMA steps' K order) and the row scales of the CTA's shared slabs.
  uint32_t B[kNJ][16];
#pragma unroll
  for (int j = 0; j < kNJ; ++j) {
    const int kb = wi + 8 * j;
    if (kb < nkbH && g < T) {
      const __nv_bfloat16* src = P.x + size_t(g) * H + kb * 128 + 8 * t;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + 32 * p));
        B[j][4 * p] = v.x;
        B[j][4 * p + 1] = v.y;
        B[j][4 * p + 2] = v.z;
        B[j][4 * p + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) B[j][i] = 0u;
    }
  }
  const Chunk c0 = w13_chunk(P, 0, b, G);  // the shared range does not depend on the routing
  if (int(threadIdx.x) < min(4 * (c0.s1 - c0.s0), kShRows)) {
    S.sh_scale[0][threadIdx.x] = __ldg(P.sh13_scale + 4 * c0.s0 + threadIdx.x);
    S.sh_scale[1][threadIdx.x] = __ldg(P.sh13_scale + P.Is + 4 * c0.s0 + threadIdx.x);
  }
  // The shared slabs do not depend on the routing: the first of them go out
  // now, and have landed by the time the router is done.
  const int nsp = min(c0.s1 - c0.s0, kStages13);
  __syncthreads();
  if (warp == 0)
    for (int p = 0; p < nsp; ++p)
      fill13(P, M, S, stages + size_t(p) * P.stage_bytes, p, w13_item(P, S.tb, c0.s0 + p), p);
  // Then the routing tables: published by the router kernel in layer mode
  // (complete and visible past the wait), built here from the caller's
  // routing in forward mode (CTA 0 publishes them for the w2 kernel).
  pdl_wait();
  if (P.layer_mode)
    read_tables(S.tb, P);
  else if (warp == 0)
    route_tables(S.rt, S.tb, P, P.topk_ids, P.topk_w, b != 0);
  __syncthreads();
  if (!P.layer_mode && b == 0 && warp == 1) publish_tables(S.tb, P);
  const Chunk ch = w13_chunk(P, S.tb.nh, b, G);
  const int npos = ch.size();
  if (warp == 0) {
    for (int p = nsp; p < kStages13 && p < npos; ++p)
      fill13(P, M, S, stages + size_t(p) * P.stage_bytes, p, w13_item(P, S.tb, ch.item(p, n_s)), p);
    if (npos <= kStages13 && lane == 0) prefetch_w2_share(P, S.tb, b, true);
  }

  // ---- f16 activations scaled by 2^sigma (each group keeps its own copy)
  {
    uint32_t mx = 0u;
#pragma unroll
    for (int j = 0; j < kNJ; ++j)
#pragma unroll
      for (int i = 0; i < 16; ++i) mx = absmax_bf16x2(mx, B[j][i]);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (t == 0) S.xmax[q][wi][g] = mx;
    named_bar_sync(2 + q, kGW * 32);
    uint32_t rmx = 0u;
    for (int w = 0; w < kGW; ++w) rmx = max(rmx, S.xmax[q][w][g]);
    const int sg = sigma_of(rmx);
    if (wi == 0 && t == 0) S.sigma[q][g] = sg;
    const float mul = __int_as_float((sg + 127) << 23);
#pragma unroll
    for (int j = 0; j < kNJ; ++j)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const __half2 hv = __floats2half2_rn(bf16_lo(B[j][i]) * mul, bf16_hi(B[j][i]) * mul);
        B[j][i] = *reinterpret_cast<const uint32_t*>(&hv);
      }
    named_bar_sync(2 + q, kGW * 32);  // the group's sigma is visible to the group
  }

  // One slab at ring position pos: the warp's K blocks, its partial tile
  // posted to shared memory; the last warp of the group to post sums the
  // partials in warp order, refills the stage with position pos + kStages13
  // and stages h. False after a timed-out wait.
  auto run_item = [&](int pos) -> bool {
    const int it = ch.item(pos, n_s);
    const Item m = w13_item(P, S.tb, it);
    const int s = pos % kStages13;
    if (!__all_sync(0xffffffffu, wait_stage(&S.full[s], &S.lastfill[s], pos, kStages13, P))) return false;
    const char* st = stages + size_t(s) * P.stage_bytes;
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
    float4 p0;
    if (m.kind == kR13) {
      // gate rows (tile rows g) and up rows (g + 8): code boxes at 0 and 4H,
      // their scale boxes from 8H
      const char* sc = st + 8 * H;
      tile_mx<kNJ, 8>(st, g, st + 4 * H, g, 8, sc, sc + align1k(8 * (H / 32)), H / 32, wi, nkbH, B, a0);
      p0 = make_float4(a0[0], a0[1], a0[2], a0[3]);
    } else {
      // rows g < 4: gate row g of the slab (tile row g) and up row g (tile row g + 8)
      tile_s8<kNJ, 8>(st, g & 3, st + 4 * H, g & 3, 4, g < 4, wi, nkbH, B, a0, a1);
      p0 = make_float4(a0[0] + a1[0], a0[1] + a1[1], a0[2] + a1[2], a0[3] + a1[3]);
    }
    float4* part = parts + size_t(s) * kGW * 32;
    part[wi * 32 + lane] = p0;
    __threadfence_block();
    __syncwarp();
    int old = 0;
    if (lane == 0) old = atomicAdd(&S.redcnt[s], 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != kGW - 1) return true;
    // Last of the group: the stage and its partials are this warp's alone.
    __threadfence_block();
    float4 d = part[lane];
#pragma unroll
    for (int w = 1; w < kGW; ++w) {
      const float4 v = part[w * 32 + lane];
      d.x += v.x;
      d.y += v.y;
      d.z += v.z;
      d.w += v.w;
    }
    if (lane == 0) S.redcnt[s] = 0;
    __syncwarp();
    if (pos + kStages13 < npos) {
      fill13(P, M, S, stages + size_t(s) * P.stage_bytes, s, w13_item(P, S.tb, ch.item(pos + kStages13, n_s)),
             pos + kStages13);
      if (pos + kStages13 == npos - 1 && lane == 0) prefetch_w2_share(P, S.tb, b, true);
    }
    const float dg[2] = {d.x, d.y}, du[2] = {d.z, d.w};
    if (m.kind == kR13) {
      const int rl = (it - n_s - ch.r0) * 8 + g;  // row among this CTA's routed rows
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int tok = 2 * t + qq;
        if (tok < T) {
          const float inv = pow2f(-S.sigma[q][tok]);
          const float h = clamped_swiglu_f(dg[qq] * inv, du[qq] * inv, P.limit) * S.tb.w[m.li * 8 + tok] * P.tau_r;
          hst_r[tok * P.hrs + rl] = __float2half_rn(h);
        }
      }
    } else if (g < 4) {
      const int rl = m.row0 + g - 4 * ch.s0;  // row among this CTA's shared rows
      const float sg = rl < kShRows ? S.sh_scale[0][rl] : __ldg(P.sh13_scale + m.row0 + g);
      const float su = rl < kShRows ? S.sh_scale[1][rl] : __ldg(P.sh13_scale + P.Is + m.row0 + g);
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int tok = 2 * t + qq;
        if (tok < T) {
          const float inv = pow2f(-S.sigma[q][tok]);
          hst_s[tok * P.hss + rl] =
              __float2half_rn(clamped_swiglu_f(dg[qq] * sg * inv, du[qq] * su * inv, P.limit) * P.tau_s);
        }
      }
    }
    return true;
  };

  // ---- item loop: group q takes ring positions q, q + 2, ... (shared slabs
  // first, then routed)
  bool ok = true;
  for (int pos = q; pos < npos && ok; pos += 2) ok = run_item(pos);
  // No copy may still be landing in this CTA's shared memory (possible only
  // after a timeout).
  __syncthreads();
  if (threadIdx.x == 0)
    for (int s = 0; s < kStages13; ++s)
      if (S.lastfill[s] >= 0) mbar_wait_bounded(&S.full[s], uint32_t(S.lastfill[s] / kStages13) & 1u, kBarTries);
  // The staged intermediates: routed rows of the tokens routed to the
  // expert (the w2 kernel reads no others), every shared row.
  const int nrr = (ch.r1 - ch.r0) * 8, nsr2 = (ch.s1 - ch.s0) * 4;
  for (int i = threadIdx.x; i < T * nrr; i += blockDim.x) {
    const int tok = i / nrr, f = ch.r0 * 8 + i % nrr;  // row of the flattened [nh, I] list
    const int li = f / P.I;
    if ((S.tb.mask[li] >> tok) & 1u) P.dh[(size_t(li) * T + tok) * P.I + f % P.I] = hst_r[tok * P.hrs + i % nrr];
  }
  for (int i = threadIdx.x; i < T * nsr2; i += blockDim.x) {
    const int tok = i / nsr2, r = i % nsr2;
    P.hs[size_t(tok) * P.Is + ch.s0 * 4 + r] = hst_s[tok * P.hss + r];
  }
}

// ---------------------------------------------------------------- w2 kernel

struct W2Smem {
  uint64_t full[kMaxStages2];
  int redcnt[kMaxStages2];
  int lastfill[kMaxStages2];
  float sh_scale[kShRows];  // shared-expert row scales of this CTA's output rows
  Tables tb;
};
constexpr size_t kHead2 = (sizeof(W2Smem) + 127) / 128 * 128;
constexpr int kW2Blocks = 2;  // 16-row output blocks per w2 CTA, at most
constexpr size_t kRed2 = size_t(kW2Blocks) * 16 * 32 * 16;  // float4 per lane, warp and block

// Ring position p of CTA b: output block rb = b w2_per + p / nl, expert slot
// l = p % nl (the shared expert first when there is one, then the routed list).
struct Item2 {
  int rb, l, li;  // li < 0: shared expert
};
__device__ __forceinline__ Item2 w2_item(const DecParams& P, int nl, int b, int p) {
  Item2 m;
  m.rb = b * P.w2_per + p / nl;
  m.l = p % nl;
  m.li = P.Is > 0 ? m.l - 1 : m.l;
  return m;
}

// Offset of the token rows of intermediates in a stage: after the larger of
// the shared box (16 int8 rows) and the routed code box (16 rows of I / 2
// bytes) with its scale box.
__host__ __device__ __forceinline__ int w2_hoff(int I, int Is) {
  const int sh = 16 * Is, ro = 8 * I + align1k(16 * (I / 32));
  return align1k(sh > ro ? sh : ro);
}

// Weight rows [rb * 16, +16) of the item's expert as one code box (and its
// scale box): adds their bytes to the stage's barrier without arriving (lane 0).
__device__ __forceinline__ void fill2_weights(const DecParams& P, const DecMaps& M, W2Smem& S, char* dst, int s,
                                              const Item2& m) {
  if (m.li < 0) {
    mbar_expect_tx(&S.full[s], uint32_t(16 * P.Is));
    tma_load_3d(dst, &M.shared, 0, m.rb * 16, 0, &S.full[s]);
  } else {
    const int r0 = S.tb.hit[m.li] * P.H + m.rb * 16;
    mbar_expect_tx(&S.full[s], uint32_t(16 * (P.I / 2) + 16 * (P.I / 32)));
    tma_load_3d(dst, &M.codes, 0, r0, 0, &S.full[s]);
    tma_load_2d(dst + 8 * P.I, &M.scales, 0, r0, &S.full[s]);
  }
}

// The intermediates of the expert's tokens (token t in slot t), then the
// stage's one arrival (whole warp). Only after the w13 grid is complete.
__device__ __forceinline__ void fill2_h(const DecParams& P, W2Smem& S, char* dst, int s, const Item2& m) {
  const int lane = threadIdx.x & 31;
  const bool sh = m.li < 0;
  const int K = sh ? P.Is : P.I;
  const uint32_t mask = sh ? (1u << P.T) - 1u : S.tb.mask[m.li];
  if (lane == 0) mbar_arrive_expect_tx(&S.full[s], uint32_t(__popc(mask)) * uint32_t(K * 2));
  __syncwarp();
  if (lane < P.T && ((mask >> lane) & 1u)) {
    const __half* src = sh ? P.hs + size_t(lane) * P.Is : P.dh + (size_t(m.li) * P.T + lane) * P.I;
    bulk_g2s(dst + w2_hoff(P.I, P.Is) + lane * K * 2, src, uint32_t(K * 2), &S.full[s]);
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kThreads, 1) k_dec_w2(DecParams P, const __grid_constant__ DecMaps M) {
  extern __shared__ __align__(128) char smem[];
  W2Smem& S = *reinterpret_cast<W2Smem*>(smem);
  char* stages = smem + ((smem_u32(smem) + uint32_t(kHead2) + 1023u) & ~1023u) - smem_u32(smem);
  float4* red = reinterpret_cast<float4*>(stages + size_t(P.nstages) * P.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int T = P.T, NS = P.nstages;
  const int b = int(blockIdx.x);
  const int nrb_mine = max(0, min(P.w2_per, P.H / 16 - b * P.w2_per));
  const bool has_sh = P.Is > 0;

  // row scales first: a global load waits behind the SM's copies in flight
  if (has_sh)
    for (int i = threadIdx.x; i < 16 * nrb_mine && i < kShRows; i += blockDim.x)
      S.sh_scale[i] = __ldg(P.sh2_scale + 16 * b * P.w2_per + i);
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], 1);
      S.redcnt[s] = 0;
      S.lastfill[s] = -1;
    }
    fence_mbar_init();
    // Position 0 is the shared expert of the first block: its weight rows do
    // not depend on the previous grids.
    if (has_sh && nrb_mine > 0) fill2_weights(P, M, S, stages, 0, Item2{b * P.w2_per, 0, -1});
  }
  __syncthreads();
  pdl_wait();
  read_tables(S.tb, P);
  __syncthreads();
  const int nl = S.tb.nh + (has_sh ? 1 : 0);
  const int n_items = nrb_mine * nl;
  if (warp == 0)
    for (int p = 0; p < NS && p < n_items; ++p) {
      const Item2 m = w2_item(P, nl, b, p);
      if (lane == 0) {
        S.lastfill[p] = p;
        if (!(p == 0 && has_sh)) fill2_weights(P, M, S, stages + size_t(p) * P.stage_bytes, p, m);
      }
      __syncwarp();
      fill2_h(P, S, stages + size_t(p) * P.stage_bytes, p, m);
    }
  // Position 0's shared weights were armed before the wait even if it turns
  // out there is nothing to do; give that copy its arrival so it can land.
  if (warp == 0 && n_items == 0 && has_sh && nrb_mine > 0 && lane == 0) {
    S.lastfill[0] = 0;
    mbar_arrive(&S.full[0]);
  }

  // Two groups of eight warps take alternate ring positions (group q the
  // positions q, q + 2, ... of the CTA's blocks x experts); warp i of a group
  // owns K blocks i, i + 8. Every warp keeps its partial sums per output
  // block in registers; once all positions are done the sixteen warps'
  // partials of each block are summed in warp order.
  const int q = warp >> 3, wi = warp & 7;
  bool ok = true;
  float4 acc[kW2Blocks];
#pragma unroll
  for (int i = 0; i < kW2Blocks; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int pos = q; pos < n_items; pos += 2) {
    const Item2 m = w2_item(P, nl, b, pos);
    const int s = pos % NS;
    // A timed-out warp keeps going (without reading the stage) so that every
    // warp reaches the final barriers.
    ok = ok && __all_sync(0xffffffffu, wait_stage(&S.full[s], &S.lastfill[s], pos, NS, P));
    if (!ok) continue;
    const char* st = stages + size_t(s) * P.stage_bytes;
    const bool sh = m.li < 0;
    const int K = sh ? P.Is : P.I;
    const int nkb = K / 128;
    const int rr = m.rb - b * P.w2_per;  // block within this CTA's
    // B: the intermediates of token g (zero for tokens not routed here)
    const uint32_t mask = sh ? (1u << T) - 1u : S.tb.mask[m.li];
    const bool has_tok = g < T && ((mask >> g) & 1u);
    uint32_t Bf[2][16];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int kb = wi + 8 * j;
      if (has_tok && kb < nkb) {
        load_b_smem(st + w2_hoff(P.I, P.Is) + g * K * 2, kb, Bf[j]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) Bf[j][i] = 0u;
      }
    }
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
    float4 d;
    if (sh) {
      tile_s8<2, 8>(st, g, st, g + 8, 16, true, wi, nkb, Bf, a0, a1);
      const int rl = rr * 16 + g;  // row within this CTA's output rows
      const float its = 1.0f / P.tau_s;
      const float sa = (rl < kShRows ? S.sh_scale[rl] : __ldg(P.sh2_scale + m.rb * 16 + g)) * its;
      const float sb = (rl + 8 < kShRows ? S.sh_scale[rl + 8] : __ldg(P.sh2_scale + m.rb * 16 + g + 8)) * its;
      d = make_float4((a0[0] + a1[0]) * sa, (a0[1] + a1[1]) * sa, (a0[2] + a1[2]) * sb, (a0[3] + a1[3]) * sb);
    } else {
      const char* sc = st + 8 * P.I;  // the scale box after the 16-row code box
      tile_mx<2, 8>(st, g, st, g + 8, 16, sc, sc, P.I / 32, wi, nkb, Bf, a0);
      const float itr = 1.0f / P.tau_r;
      d = make_float4(a0[0] * itr, a0[1] * itr, a0[2] * itr, a0[3] * itr);
    }
#pragma unroll
    for (int i = 0; i < kW2Blocks; ++i)
      if (i == rr) {
        acc[i].x += d.x;
        acc[i].y += d.y;
        acc[i].z += d.z;
        acc[i].w += d.w;
      }
    // the last warp of the group to finish with the stage refills it
    __syncwarp();
    int old = 0;
    if (lane == 0) old = atomicAdd(&S.redcnt[s], 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old == 7) {
      if (lane == 0) S.redcnt[s] = 0;
      __syncwarp();
      const int np = pos + NS;
      if (np < n_items) {
        const Item2 mn = w2_item(P, nl, b, np);
        if (lane == 0) {
          S.lastfill[s] = np;
          fill2_weights(P, M, S, stages + size_t(s) * P.stage_bytes, s, mn);
        }
        __syncwarp();
        fill2_h(P, S, stages + size_t(s) * P.stage_bytes, s, mn);
      }
    }
  }
  // every block: the sixteen warps' partials summed in warp order, bf16
#pragma unroll
  for (int i = 0; i < kW2Blocks; ++i) red[(i * 16 + warp) * 32 + lane] = acc[i];
  __syncthreads();
  if (warp < nrb_mine) {
    const int r = warp;
    float4 d = red[(r * 16) * 32 + lane];
    for (int w = 1; w < 16; ++w) {
      const float4 v = red[(r * 16 + w) * 32 + lane];
      d.x += v.x;
      d.y += v.y;
      d.z += v.z;
      d.w += v.w;
    }
    const float v[4] = {d.x, d.y, d.z, d.w};
    const int rb = b * P.w2_per + r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = 2 * t + (i & 1);
      if (tok < T) P.out[size_t(tok) * P.H + rb * 16 + g + 8 * (i >> 1)] = __float2bfloat16_rn(v[i]);
    }
  }
  // No copy may still be landing in this CTA's shared memory.
  __syncthreads();
  if (threadIdx.x == 0)
    for (int s = 0; s < NS; ++s)
      if (S.lastfill[s] >= 0) mbar_wait_bounded(&S.full[s], uint32_t(S.lastfill[s] / NS) & 1u, kBarTries);
}

// ---------------------------------------------------------------- host side

// 2^e for the largest e <= 14 with bound * 2^e below the f16 maximum.
float h_scale(float bound) {
  int e = 0;
  while (e < 14 && bound * std::ldexp(1.0f, e + 1) < 65504.0f) ++e;
  return std::ldexp(1.0f, e);
}

struct Plan {
  int stage13 = 0, stage2 = 0, nst2 = 0, hrs = 0, hss = 0;
  size_t smem13 = 0, smem2 = 0;
  bool ok = false;
};

size_t route_smem_bytes(const v4moe_config& c, int T) {
  return kRouteTail + (size_t(T) * c.n_experts + c.n_experts) * 4 + 16 + size_t(T) * c.hidden * 2;
}

// Router cluster size: the largest of 16, 8, 4, 2 CTAs (at most one per 16
// experts' warps) that the device can co-schedule with this shared memory;
// queried once per device and size class. 0 if none.
int route_cluster(size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaFuncSetAttribute(k_dec_route, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  int best = 0;
  for (int cl = kRouteMaxCluster; cl >= 2 && best == 0; cl /= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl);
    cfg.blockDim = dim3(kRouteWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(cl);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_dec_route, &cfg) == cudaSuccess && n >= 1) best = cl;
  }
  cudaGetLastError();  // a refused size leaves no sticky error
  cache[key] = best;
  return best;
}

Plan make_plan(const v4moe_config& c, int T, int G) {
  Plan p;
  if (T < 1 || T > kDecodeMaxTokens || T * c.top_k > kMaxHit) return p;
  const int H = c.hidden, I = c.inter, Is = c.shared_inter;
  if (H > kNJ * 8 * 128 || I > 2 * 8 * 128 || Is > 2 * 8 * 128) return p;
  // Scale rows of K / 32 bytes: a swizzle span (16 .. 128 bytes), so K is a
  // power of two from 512; shared rows whole 128-byte chunks.
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  if (H % 512 != 0 || I % 512 != 0 || !pow2(H) || !pow2(I) || Is % 128 != 0) return p;
  const int s13 = std::max(8 * H + 2 * align1k(8 * (H / 32)), Is > 0 ? 8 * H : 0);
  p.stage13 = align1k(s13);
  // staged intermediates: a CTA's share of the routed rows (at most
  // min(E, T k) experts hit) and of the shared rows, per token
  const int nh_max = std::min(c.n_experts, T * c.top_k);
  p.hrs = (nh_max * (I / 8) + G - 1) / G * 8;
  p.hss = (Is / 4 + G - 1) / G * 4;
  const size_t hstage = size_t(T) * (p.hrs + p.hss) * 2;
  // 1024 bytes of slack put the first stage on a multiple of 1024
  p.smem13 = kHead13 + 1024 + size_t(kStages13) * p.stage13 + kPart13 + (hstage + 127) / 128 * 128;
  p.stage2 = align1k(w2_hoff(I, Is) + T * std::max(I, Is) * 2);
  const size_t room = 227 * 1024 - kHead2 - 1024 - kRed2;
  p.nst2 = int(std::min<size_t>(kMaxStages2, room / p.stage2));
  p.smem2 = kHead2 + 1024 + size_t(p.nst2) * p.stage2 + kRed2;
  p.ok = p.smem13 <= 227 * 1024 && p.nst2 >= 2 && route_smem_bytes(c, T) <= 227 * 1024 &&
         (H / 16 + G - 1) / G <= kW2Blocks;
  return p;
}

// u8 maps of the weights the slab kernels stream (see DecMaps). False when a
// map cannot be encoded (a base address off 16 bytes).
bool dec_maps(const v4moe_config& c, const v4moe_weights& w, DecMaps& m13, DecMaps& m2) {
  const uint64_t H = c.hidden, I = c.inter, Is = c.shared_inter, E = c.n_experts;
  auto chunked = [](CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
    const uint64_t dims[3] = {128, rows, row_bytes / 128};
    const uint64_t strides[2] = {row_bytes, 128};
    const uint32_t box[3] = {128, box_rows, uint32_t(row_bytes / 128)};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B);
  };
  auto scales = [](CUtensorMap* m, const void* base, uint64_t rows, uint64_t S, uint32_t box_rows) {
    const uint64_t dims[2] = {S, rows};
    const uint64_t strides[1] = {S};
    const uint32_t box[2] = {uint32_t(S), box_rows};
    const CUtensorMapSwizzle sw = S >= 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : S == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : S == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, sw);
  };
  m13 = DecMaps{};
  m2 = DecMaps{};
  bool ok = chunked(&m13.codes, w.w13_codes, E * 2 * I, H / 2, 8) && scales(&m13.scales, w.w13_scales, E * 2 * I, H / 32, 8) &&
            chunked(&m2.codes, w.w2_codes, E * H, I / 2, 16) && scales(&m2.scales, w.w2_scales, E * H, I / 32, 16);
  if (ok && Is > 0)
    ok = chunked(&m13.shared, w.sh_w13, 2 * Is, H, 4) && chunked(&m2.shared, w.sh_w2, H, Is, 16);
  return ok;
}

}  // namespace

DecodeBuffers dec_buffers(const v4moe_config& c, int64_t T) {
  DecodeBuffers b;
  if (T < 1 || T > kDecodeMaxTokens) return b;
  b.ctl = size_t(cWords) * 4;
  b.dh = size_t(kMaxHit) * T * c.inter * 2;
  b.hs = size_t(T) * std::max(c.shared_inter, 0) * 2;
  return b;
}

bool dec_supported(const v4moe_config& c, int T) { return make_plan(c, T, device_sms()).ok; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  const v4moe_config& c = a.c;
  const int sms = device_sms();
  const Plan p = make_plan(c, a.T, sms);
  if (!p.ok) return cudaErrorInvalidValue;
  DecMaps m13, m2;
  if (!dec_maps(c, a.w, m13, m2)) return cudaErrorInvalidValue;
  DecParams P;
  P.T = a.T;
  P.H = c.hidden;
  P.I = c.inter;
  P.Is = c.shared_inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.vocab = c.vocab;
  P.limit = c.swiglu_limit;
  P.routed_scale = c.routed_scale;
  // |h| <= L * L * |routed_scale| (routed weights sum to routed_scale) and
  // L * L (shared): the largest power of two that keeps h * tau below the f16
  // maximum gives small intermediates that many more binades
  const float L = c.swiglu_limit;
  P.tau_r = h_scale(L * L * std::max(1.0f, std::fabs(c.routed_scale)));
  P.tau_s = h_scale(L * L);
  P.layer_mode = a.layer_mode;
  P.stage_bytes = 0;
  P.nstages = 0;
  P.w2_per = 1;
  P.hrs = p.hrs;
  P.hss = p.hss;
  P.x = a.x;
  P.gate = a.gate;
  P.bias = a.bias;
  P.token_ids = a.token_ids;
  P.tid2eid = a.tid2eid;
  P.topk_ids = a.topk_ids;
  P.topk_w = a.topk_w;
  P.counts = a.counts;
  P.offsets = a.offsets;
  P.sorted_slot = a.sorted_slot;
  P.slot_pos = a.slot_pos;
  P.w13_codes = a.w.w13_codes;
  P.w13_scales = a.w.w13_scales;
  P.w2_codes = a.w.w2_codes;
  P.w2_scales = a.w.w2_scales;
  P.sh13 = a.w.sh_w13;
  P.sh13_scale = a.w.sh_w13_scale;
  P.sh2 = a.w.sh_w2;
  P.sh2_scale = a.w.sh_w2_scale;
  P.dh = a.dh;
  P.hs = a.hs;
  P.ctl = a.ctl;
  P.status = a.status;
  P.out = a.out;

  const int nrb = c.hidden / 16;
  P.w2_per = (nrb + sms - 1) / sms;
  const int grid2 = (nrb + P.w2_per - 1) / P.w2_per;
  cudaError_t e = cudaSuccess;
  if (a.layer_mode) {
    const size_t route_smem = route_smem_bytes(c, a.T);
    set_smem(k_dec_route, route_smem);
    const int cl = route_cluster(route_smem);
    if (cl <= 0) return cudaErrorInvalidValue;
    e = launch_kernel_cl("dec_route", k_dec_route, dim3(cl), dim3(kRouteWarps * 32), route_smem, st, false, cl, P);
    if (e != cudaSuccess) return e;
  }
  // Without a routing kernel in front, the w13 kernel must not overlap the
  // previous call's w2 kernel (it rewrites the intermediates that one reads).
  P.stage_bytes = p.stage13;
  set_smem(k_dec_w13, p.smem13);
  e = launch_kernel("dec_w13", k_dec_w13, dim3(sms), dim3(kThreads), p.smem13, st, a.layer_mode != 0, P, m13);
  if (e != cudaSuccess) return e;
  P.stage_bytes = p.stage2;
  P.nstages = p.nst2;
  set_smem(k_dec_w2, p.smem2);
  return launch_kernel("dec_w2", k_dec_w2, dim3(grid2), dim3(kThreads), p.smem2, st, true, P, m2);
}

}  // namespace v4moe
