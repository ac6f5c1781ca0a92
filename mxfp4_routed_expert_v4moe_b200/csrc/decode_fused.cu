// Decode-sized batches (at most 8 tokens): the whole layer in ONE persistent
// kernel that streams every weight byte once.
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
// One CTA per SM, three warp roles:
//  * 16 consumer warps multiply the weight tile of each ring slot with
//    mma.sync m16n8k16 (f16 operands, fp32 accumulation, the tokens as the 8
//    columns): E2M1 pairs via cvt and int8 via a magic-number conversion,
//    both exact; each warp owns two 128-wide K blocks of the tile and posts
//    its partial tile; the last warp to post adds the partials in warp order
//    and runs the slot's epilogue.
//  * a producer warp fills the ring with 1-D bulk copies, in the CTA's item
//    order: its gate rows, its share of the shared expert's w13 rows, then
//    (once the routing is known) its shares of the routed w13 slabs, of the
//    shared expert's w2 rows and of the routed w2 rows.
//  * a control warp: the routing (waits until every CTA has posted its router
//    scores, selects each token's experts, builds the tables and the CTA's
//    ranges), the routing outputs (CTA 0), and the copy of the intermediates
//    h that the CTA's w2 rows multiply, once the CTAs computing them are done.
//
// Data crosses CTAs through global memory only, with counters in the
// workspace's control block: router arrivals, finished w13 slabs per expert,
// and w2 partial sums per 16-row output block. The w2 rows are shared out
// expert by expert (a CTA holds the rows of one or two experts), so every
// output block gets one partial sum per expert in a workspace slot; the last
// CTA to post a block's partial adds the slots in expert order (shared expert
// first, then ascending expert id) and writes bf16 out, so the result does
// not depend on timing. The last CTA to finish resets the counters.
//
// The intermediates are stored as f16 scaled by a fixed power of two chosen
// from the clamp limit: |h| <= L * L * routed_scale, so h * 2^tau stays below
// the f16 maximum for every input while small values keep that many more
// binades.
//
// Every wait is bounded; a wait that gives up sets the status word's timeout
// bit, and the CTA stops, waits (bounded) for its own copies in flight and
// returns. Word 1 of the status block, when non-zero, makes the router wait
// expect one arrival more than there are CTAs and sets its iteration limit:
// the test of that path.
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

constexpr int kFW = 16;                    // consumer warps
constexpr int kProd = kFW;                 // producer warp
constexpr int kCtl = kFW + 1;              // control warp
constexpr int kFThreads = (kFW + 2) * 32;
constexpr int kMaxSlots = 8;
constexpr int kFMaxHit = 64;               // distinct routed experts (T * k <= 64)
constexpr int kMaxGateRows = 4;            // gate rows per CTA
constexpr int kMaxHSlots = 4;              // experts whose w2 rows one CTA holds
constexpr uint32_t kWaitTries = 1u << 22;  // mbarrier try_wait rounds
constexpr uint32_t kPollTries = 1u << 20;  // global-counter polls (each sleeps)

// Control block (workspace, uint32 words; zero at rest).
enum FCtl : int {
  fRoute = 0,                 // router arrivals (one per CTA)
  fExit = 1,                  // CTAs finished
  fH = 16,                    // [kFMaxHit + 1] finished w13 slabs per expert list index
  fBlk = fH + kFMaxHit + 16,  // [H / 16] w2 partials posted per 16-row output block
  fWords = fBlk + 256,
};

enum FKind : int { iNone = 0, iGate = 1, iS13 = 2, iR13 = 3, iS2 = 4, iR2 = 5 };

struct FParams {
  int T, H, I, Is, E, k, vocab;
  float limit, routed_scale;
  float tau_r, tau_s;  // 2^tau: routed / shared intermediate scales
  int layer_mode;
  int nslots, slot_bytes;
  int hbuf_bytes;      // one intermediate staging buffer: T * max(I, Is) f16
  int G;               // grid size
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
  float* scores;  // [T, E]
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  const int8_t* sh13;
  const float* sh13_scale;
  const int8_t* sh2;
  const float* sh2_scale;
  __half* dh;    // [kFMaxHit + 1][T][max(I, Is)]: list index 0 = shared expert
  float* part;   // [kFMaxHit + 1][H][T] w2 partial sums
  uint32_t* ctl;
  uint32_t* status;
  __nv_bfloat16* out;
};

// A contiguous share of a list of n items for CTA b of G: every CTA gets
// n / G items, and the n % G extra ones go to the CTAs of the cyclic interval
// [a, a + n % G), so that the extras of successive lists land on different
// CTAs.
struct Share {
  int lo, hi;
};
__host__ __device__ __forceinline__ Share share_of(int n, int G, int a, int b) {
  const int base = n / G, e = n % G;
  int before;  // extras among CTAs [0, b)
  if (a + e <= G)
    before = min(max(b - a, 0), e);
  else
    before = min(b, a + e - G) + max(0, b - a);
  const bool extra = ((b - a + G) % G) < e;
  Share s;
  s.lo = b * base + before;
  s.hi = s.lo + base + (extra ? 1 : 0);
  return s;
}

// The CTA's ranges of the four item lists: shared w13 slabs (4 channels: 4
// gate + 4 up rows), shared w2 units (16 output rows), routed w13 slabs (8
// channels of one expert) and routed w2 units (32 output rows of one expert);
// the routed lists run expert by expert in ascending id.
struct Work {
  Share a, c, bq, d;  // sh13, sh2, r13, r2
};
__host__ __device__ __forceinline__ Work work_split(int Is, int H, int I, int G, int nh, int b) {
  Work w;
  const int n_a = Is > 0 ? Is / 4 : 0, n_c = Is > 0 ? H / 16 : 0, n_b = nh * (I / 8), n_d = nh * (H / 32);
  int a = 0;
  w.a = share_of(n_a, G, a, b);
  a = (a + n_a % G) % G;
  w.c = share_of(n_c, G, a, b);
  a = (a + n_c % G) % G;
  w.bq = share_of(n_b, G, a, b);
  a = (a + n_b % G) % G;
  w.d = share_of(n_d, G, a, b);
  return w;
}

struct FItem {
  int kind, l, row0, e;  // l: expert list index (0 = shared); row0: first channel / output row
};

struct FSmem {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t hfull[2];
  uint64_t hfree[2];
  int redcnt[kMaxSlots];
  int ready;     // tables and ranges valid
  int abort_;    // a bounded wait gave up
  int ng, e0;    // gate rows of this CTA
  int npos_pre;  // positions that need no routing
  int npos;      // all positions (valid once ready)
  int nhl;       // experts whose intermediates the w2 units read
  int hl[kMaxHSlots];
  int sigma[8];
  uint32_t xmax[kFW][8];
  Work w;
  int nh;
  int hit[kFMaxHit];
  uint32_t mask[kFMaxHit];
  float tw[kFMaxHit * 8];
  uint32_t bits[32];
  int rank_base[32];
  int cnt[kFMaxHit];
  int cum[kFMaxHit + 1];
  int ids[64];
  float wts[64];
  int32_t sel_ids[64];
  float sel_w[64];
  float gp[kFW][kMaxGateRows * 8];
};

constexpr size_t kFHead = (sizeof(FSmem) + 127) / 128 * 128;

__device__ __forceinline__ float pow2f_(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((e + 127) << 23);
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool aborted(FSmem& S) { return *reinterpret_cast<volatile int*>(&S.abort_) != 0; }

__device__ __forceinline__ void set_abort(FSmem& S, const FParams& P) {
  atomicOr(P.status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(&S.abort_) = 1;
}

// Bounded wait on an mbarrier phase; gives up early once the CTA aborts.
__device__ __forceinline__ bool fwait(FSmem& S, uint64_t* bar, uint32_t parity, const FParams& P) {
  for (uint32_t i = 0; i < kWaitTries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15) == 15 && aborted(S)) return false;
  }
  set_abort(S, P);
  return false;
}

// Bounded poll of a global counter until it reaches `target`.
__device__ __forceinline__ bool fpoll(FSmem& S, const uint32_t* p, uint32_t target, uint32_t tries,
                                      const FParams& P) {
  for (uint32_t i = 0; i < tries; ++i) {
    if (ld_acquire(p) >= target) return true;
    if (aborted(S)) return false;
    __nanosleep(64);
  }
  set_abort(S, P);
  return false;
}

// Waits (bounded) until the control warp has published the tables.
__device__ __forceinline__ bool wait_ready(FSmem& S) {
  for (uint32_t i = 0; i < kPollTries * 64; ++i) {
    if (*reinterpret_cast<volatile int*>(&S.ready)) {
      __threadfence_block();
      return true;
    }
    if (aborted(S)) return false;
    __nanosleep(32);
  }
  return false;
}

// ---------------------------------------------------------------- tiles

// B fragment (16 words: token g's f16 elements kb * 128 + 32 t .. + 31 of K
// block kb) from shared memory; src is null for a column past the batch.
__device__ __forceinline__ void load_b(const char* src, uint32_t (&B)[16]) {
  if (src) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = s4[q];
      B[4 * q] = v.x;
      B[4 * q + 1] = v.y;
      B[4 * q + 2] = v.z;
      B[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) B[i] = 0u;
  }
}

// MXFP4 m16 tile: rows g and g + 8 at ra / rb (codes of 128-wide K block kb at
// kb * 64), their E8M0 scale rows at sa / sb. The warp's K blocks kb = kb0 +
// KS j (j < NJ, kb < nkb) multiply the B fragments bsrc(kb) gives. The group
// scales enter the f16 operand as powers of two relative to the largest
// exponent of the row among the warp's groups (f16 operands stay below
// 6 * 2^13); fa / fb get the rest.
template <int NJ, int KS, class BSrc>
__device__ __forceinline__ void ftile_mx(const char* ra, const char* rb, const uint8_t* sa, const uint8_t* sb,
                                         int kb0, int nkb, BSrc bsrc, float (&ae)[4], float (&ao)[4], float& fa,
                                         float& fb) {
  const int t = threadIdx.x & 3;
  int xa = 0, xb = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int kb = kb0 + KS * j;
    if (kb < nkb) {
      xa = max(xa, int(sa[4 * kb + t]));
      xb = max(xb, int(sb[4 * kb + t]));
    }
  }
  xa = max(xa, __shfl_xor_sync(0xffffffffu, xa, 1));
  xa = max(xa, __shfl_xor_sync(0xffffffffu, xa, 2));
  xb = max(xb, __shfl_xor_sync(0xffffffffu, xb, 1));
  xb = max(xb, __shfl_xor_sync(0xffffffffu, xb, 2));
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int kb = kb0 + KS * j;
    if (kb < nkb) {
      uint32_t B[16];
      load_b(bsrc(kb), B);
      const uint4 qa = *reinterpret_cast<const uint4*>(ra + kb * 64 + 16 * t);
      const uint4 qb = *reinterpret_cast<const uint4*>(rb + kb * 64 + 16 * t);
      const uint32_t fsa = f16_pow2_bits(int(sa[4 * kb + t]) - xa + 13) * 0x10001u;
      const uint32_t fsb = f16_pow2_bits(int(sb[4 * kb + t]) - xb + 13) * 0x10001u;
      const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
      const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t ca[4], cb[4];
        e2m1x8_to_f16x2(wa[u], ca);
        e2m1x8_to_f16x2(wb[u], cb);
        const uint32_t A0[4] = {hmul2_u32(ca[0], fsa), hmul2_u32(cb[0], fsb), hmul2_u32(ca[1], fsa),
                                hmul2_u32(cb[1], fsb)};
        const uint32_t A1[4] = {hmul2_u32(ca[2], fsa), hmul2_u32(cb[2], fsb), hmul2_u32(ca[3], fsa),
                                hmul2_u32(cb[3], fsb)};
        mma_16816_f16(ae, A0, B[4 * u], B[4 * u + 1]);
        mma_16816_f16(ao, A1, B[4 * u + 2], B[4 * u + 3]);
      }
    }
  }
  fa = pow2f_(xa - 127 - 13);
  fb = pow2f_(xb - 127 - 13);
}

// int8 m16 tile: rows g and g + 8 at ra / rb (K block kb at kb * 128), zero
// rows where `valid` is false; the warp's K blocks kb = kb0 + KS j < nkb.
template <int NJ, int KS, class BSrc>
__device__ __forceinline__ void ftile_s8(const char* ra, const char* rb, bool valid, int kb0, int nkb, BSrc bsrc,
                                         float (&ae)[4], float (&ao)[4]) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int kb = kb0 + KS * j;
    if (kb < nkb) {
      uint32_t B[16];
      load_b(bsrc(kb), B);
      uint4 qa0 = make_uint4(0u, 0u, 0u, 0u), qa1 = qa0, qb0 = qa0, qb1 = qa0;
      if (valid) {
        const char* pa = ra + kb * 128 + 32 * t;
        const char* pb = rb + kb * 128 + 32 * t;
        qa0 = *reinterpret_cast<const uint4*>(pa);
        qa1 = *reinterpret_cast<const uint4*>(pa + 16);
        qb0 = *reinterpret_cast<const uint4*>(pb);
        qb1 = *reinterpret_cast<const uint4*>(pb + 16);
      }
      const uint32_t wa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
      const uint32_t wb[8] = {qb0.x, qb0.y, qb0.z, qb0.w, qb1.x, qb1.y, qb1.z, qb1.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t A[4];
        s8x4_to_f16x2(wa[s], A[0], A[2]);
        s8x4_to_f16x2(wb[s], A[1], A[3]);
        if (s & 1)
          mma_16816_f16(ao, A, B[2 * s], B[2 * s + 1]);
        else
          mma_16816_f16(ae, A, B[2 * s], B[2 * s + 1]);
      }
    }
  }
}

// ---------------------------------------------------------------- items

// Item at ring position p of this CTA. Order: the gate rows (one item, layer
// mode), shared w13 slabs, then -- with the tables -- routed w13 slabs,
// shared w2 units, routed w2 units.
__device__ __forceinline__ FItem item_at(const FParams& P, const FSmem& S, int p) {
  FItem m = {iNone, 0, 0, 0};
  if (S.ng > 0) {
    if (p == 0) {
      m.kind = iGate;
      return m;
    }
    --p;
  }
  const Work& w = S.w;
  const int na = w.a.hi - w.a.lo;
  if (p < na) {
    m.kind = iS13;
    m.row0 = 4 * (w.a.lo + p);
    return m;
  }
  p -= na;
  const int nb = w.bq.hi - w.bq.lo;
  if (p < nb) {
    const int r = w.bq.lo + p, per = P.I / 8;
    m.kind = iR13;
    m.l = 1 + r / per;
    m.row0 = 8 * (r % per);
    m.e = S.hit[m.l - 1];
    return m;
  }
  p -= nb;
  const int nc = w.c.hi - w.c.lo;
  if (p < nc) {
    m.kind = iS2;
    m.row0 = 16 * (w.c.lo + p);
    return m;
  }
  p -= nc;
  const int nd = w.d.hi - w.d.lo;
  if (p < nd) {
    const int r = w.d.lo + p, per = P.H / 32;
    m.kind = iR2;
    m.l = 1 + r / per;
    m.row0 = 32 * (r % per);
    m.e = S.hit[m.l - 1];
  }
  return m;
}

__host__ __device__ __forceinline__ uint32_t bytes_s13(int H) { return uint32_t(8 * H + 32); }
__host__ __device__ __forceinline__ uint32_t bytes_r13(int H) { return uint32_t(16 * (H / 2) + 16 * (H / 32)); }
__host__ __device__ __forceinline__ uint32_t bytes_s2(int Is) { return uint32_t(16 * Is + 64); }
__host__ __device__ __forceinline__ uint32_t bytes_r2(int I) { return uint32_t(32 * (I / 2) + 32 * (I / 32)); }

// Issue the bulk copies of item m into slot s (one lane).
__device__ __forceinline__ void issue_item(const FParams& P, FSmem& S, char* dst, int s, const FItem& m) {
  uint64_t* bar = &S.full[s];
  const int H = P.H;
  switch (m.kind) {
    case iGate:
      mbar_arrive_expect_tx(bar, uint32_t(S.ng) * H * 2);
      bulk_g2s(dst, P.gate + size_t(S.e0) * H, uint32_t(S.ng) * H * 2, bar);
      break;
    case iS13: {
      mbar_arrive_expect_tx(bar, bytes_s13(H));
      const char* sh = reinterpret_cast<const char*>(P.sh13);
      bulk_g2s(dst, sh + size_t(m.row0) * H, uint32_t(4 * H), bar);
      bulk_g2s(dst + 4 * H, sh + size_t(P.Is + m.row0) * H, uint32_t(4 * H), bar);
      bulk_g2s(dst + 8 * H, P.sh13_scale + m.row0, 16u, bar);
      bulk_g2s(dst + 8 * H + 16, P.sh13_scale + P.Is + m.row0, 16u, bar);
      break;
    }
    case iR13: {
      mbar_arrive_expect_tx(bar, bytes_r13(H));
      const size_t rg = size_t(m.e) * 2 * P.I + m.row0, ru = rg + P.I;
      bulk_g2s(dst, P.w13_codes + rg * (H / 2), uint32_t(8 * (H / 2)), bar);
      bulk_g2s(dst + 8 * (H / 2), P.w13_codes + ru * (H / 2), uint32_t(8 * (H / 2)), bar);
      bulk_g2s(dst + 16 * (H / 2), P.w13_scales + rg * (H / 32), uint32_t(8 * (H / 32)), bar);
      bulk_g2s(dst + 16 * (H / 2) + 8 * (H / 32), P.w13_scales + ru * (H / 32), uint32_t(8 * (H / 32)), bar);
      break;
    }
    case iS2:
      mbar_arrive_expect_tx(bar, bytes_s2(P.Is));
      bulk_g2s(dst, reinterpret_cast<const char*>(P.sh2) + size_t(m.row0) * P.Is, uint32_t(16 * P.Is), bar);
      bulk_g2s(dst + 16 * P.Is, P.sh2_scale + m.row0, 64u, bar);
      break;
    case iR2: {
      mbar_arrive_expect_tx(bar, bytes_r2(P.I));
      const size_t r0 = size_t(m.e) * H + m.row0;
      bulk_g2s(dst, P.w2_codes + r0 * (P.I / 2), uint32_t(32 * (P.I / 2)), bar);
      bulk_g2s(dst + 32 * (P.I / 2), P.w2_scales + r0 * (P.I / 32), uint32_t(32 * (P.I / 32)), bar);
      break;
    }
  }
}

// ---------------------------------------------------------------- routing (control warp)

// Distinct routed experts in ascending id, per (expert, token) weights and
// token masks, from the k ids / weights of each token (shared memory).
__device__ __forceinline__ void build_tables(FSmem& S, const FParams& P, bool quiet) {
  const int lane = threadIdx.x & 31;
  const int Sn = P.T * P.k;
  S.bits[lane] = 0u;
  __syncwarp();
  bool bad = false;
  for (int s = lane; s < 64; s += 32) {
    int e = -1;
    float w = 0.f;
    if (s < Sn) {
      e = S.sel_ids[s];
      w = S.sel_w[s];
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
  for (int i = lane; i < kFMaxHit * 8; i += 32) S.tw[i] = 0.f;
  for (int i = lane; i < kFMaxHit; i += 32) {
    S.mask[i] = 0u;
    S.cnt[i] = 0;
  }
  __syncwarp();
  for (int s = lane; s < Sn; s += 32) {
    const int e = S.ids[s];
    if (e >= 0) {
      const int r = S.rank_base[e >> 5] + __popc(S.bits[e >> 5] & ((1u << (e & 31)) - 1u));
      const int tok = s / P.k;
      S.hit[r] = e;
      atomicAdd(&S.tw[r * 8 + tok], S.wts[s]);
      atomicOr(&S.mask[r], 1u << tok);
      atomicAdd(&S.cnt[r], 1);
    }
  }
  if (lane == 0) S.nh = nh;
  __syncwarp();
}

// Stable counting sort of the batch's slots by expert (layer-mode outputs),
// from the state build_tables left; one warp.
__device__ __forceinline__ void write_perm(FSmem& S, const FParams& P) {
  const int lane = threadIdx.x & 31;
  const int nh = S.nh;
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
  if (lane == 0) S.cum[kFMaxHit] = total;
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

// Adds the partial sums of output block rb (16 rows) over the expert slots in
// list order and writes bf16 out (lanes g, t < tq of the calling warp), then
// clears the block's counter.
__device__ __forceinline__ void finish_block(const FParams& P, int rb, int l0, int nl_end) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int T = P.T;
  __threadfence();
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int row = rb * 16 + g + 8 * hh;
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      const int tok = 2 * t + qq;
      if (tok < T) {
        float s = 0.f;
        for (int l = l0; l < nl_end; ++l) s += __ldcg(P.part + (size_t(l) * P.H + row) * T + tok);
        P.out[size_t(tok) * P.H + row] = __float2bfloat16_rn(s);
      }
    }
  }
  __syncwarp();
  if (lane == 0) P.ctl[fBlk + rb] = 0u;
}

// Posts rows [row0, row0 + 16) of expert slot l (values v: rows g and g + 8,
// tokens 2t and 2t + 1) and counts the block's arrival; the last arrival
// finishes the block.
__device__ __forceinline__ void post_block(const FParams& P, int l, int row0, const float (&v)[4], int nl,
                                           int l0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int T = P.T;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh)
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      const int tok = 2 * t + qq;
      if (tok < T) P.part[(size_t(l) * P.H + row0 + g + 8 * hh) * T + tok] = v[2 * hh + qq];
    }
  __threadfence();
  __syncwarp();
  uint32_t old = 0;
  if (lane == 0) old = atomicAdd(P.ctl + fBlk + row0 / 16, 1u);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old == uint32_t(nl) - 1u) finish_block(P, row0 / 16, l0, l0 + nl);
}

// Epilogue of ring slot s holding item m (the last consumer warp to post):
// sums the 16 partial tiles in warp order (routed w2 units: warps 0-7 and
// 8-15 for their two 16-row tiles), releases the slot to the producer and
// writes the item's results.
__device__ __forceinline__ void epilogue(const FParams& P, FSmem& S, const FItem& m, const char* st,
                                         const float4* part, int s, int tq, int lsh) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int T = P.T, H = P.H;
  if (m.kind == iGate) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[s]);
    if (lane < S.ng * T) {
      const int r = lane / T, tok = lane % T;
      float z = 0.f;
      for (int w = 0; w < kFW; ++w) z += S.gp[w][r * 8 + tok];
      P.scores[size_t(tok) * P.E + S.e0 + r] = sqrt_softplus_f(z * pow2f_(-S.sigma[tok]));
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(P.ctl + fRoute, 1u);
    return;
  }
  float4 d0 = make_float4(0.f, 0.f, 0.f, 0.f), d1 = d0;
  if (t < tq) {
    const int w1 = m.kind == iR2 ? 8 : kFW;
    for (int w = 0; w < w1; ++w) {
      const float4 v = part[(w * 8 + g) * tq + t];
      d0.x += v.x;
      d0.y += v.y;
      d0.z += v.z;
      d0.w += v.w;
    }
    if (m.kind == iR2)
      for (int w = 8; w < kFW; ++w) {
        const float4 v = part[(w * 8 + g) * tq + t];
        d1.x += v.x;
        d1.y += v.y;
        d1.z += v.z;
        d1.w += v.w;
      }
  }
  if (m.kind == iR13 || m.kind == iS13) {
    const bool sh = m.kind == iS13;
    float sgs = 1.f, sus = 1.f;
    if (sh && g < 4) {
      sgs = reinterpret_cast<const float*>(st + 8 * H)[g];
      sus = reinterpret_cast<const float*>(st + 8 * H + 16)[g];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[s]);
    const uint32_t mask = sh ? 0xFFu : S.mask[m.l - 1];
    const int l = sh ? 0 : m.l;
    const float tau = sh ? P.tau_s : P.tau_r;
    const float dv[4] = {d0.x, d0.y, d0.z, d0.w};
    if (t < tq && (!sh || g < 4)) {
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int tok = 2 * t + qq;
        if (tok < T && ((mask >> tok) & 1u)) {
          const float inv = pow2f_(-S.sigma[tok]);
          float h = clamped_swiglu_f(dv[qq] * sgs * inv, dv[2 + qq] * sus * inv, P.limit) * tau;
          if (!sh) h *= S.tw[(m.l - 1) * 8 + tok];
          P.dh[(size_t(l) * T + tok) * max(P.I, P.Is) + m.row0 + g] = __float2half_rn(h);
        }
      }
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(P.ctl + fH + l, 1u);
    return;
  }
  const int nl = (P.Is > 0 ? 1 : 0) + S.nh;
  if (m.kind == iS2) {
    const float sa = reinterpret_cast<const float*>(st + 16 * P.Is)[g];
    const float sb = reinterpret_cast<const float*>(st + 16 * P.Is)[g + 8];
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[s]);
    const float inv = 1.0f / P.tau_s;
    const float v[4] = {d0.x * sa * inv, d0.y * sa * inv, d0.z * sb * inv, d0.w * sb * inv};
    post_block(P, 0, m.row0, v, nl, lsh);
    return;
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&S.empty[s]);
  const float inv = 1.0f / P.tau_r;
  const float v0[4] = {d0.x * inv, d0.y * inv, d0.z * inv, d0.w * inv};
  const float v1[4] = {d1.x * inv, d1.y * inv, d1.z * inv, d1.w * inv};
  post_block(P, m.l, m.row0, v0, nl, lsh);
  post_block(P, m.l, m.row0 + 16, v1, nl, lsh);
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kFThreads, 1) k_dec_fused(FParams P) {
  extern __shared__ __align__(128) char smem[];
  FSmem& S = *reinterpret_cast<FSmem*>(smem);
  char* xf = smem + kFHead;                                         // x fragments (T * H f16)
  char* hbufs = xf + size_t(P.T) * P.H * 2;                         // 2 staging buffers
  char* ring = hbufs + 2 * size_t(P.hbuf_bytes);                    // nslots * slot_bytes
  const int tq = (P.T + 1) / 2;                                     // token pairs
  float4* parts = reinterpret_cast<float4*>(ring + size_t(P.nslots) * P.slot_bytes);  // [slot][warp][8][tq]
  float* ssc = reinterpret_cast<float*>(parts + size_t(P.nslots) * kFW * 8 * tq);      // scores [T][E]
  float* sbias = ssc + size_t(P.T) * P.E;                                               // [E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = P.T, H = P.H, G = P.G, b = int(blockIdx.x);
  const int NS = P.nslots;
  const bool learned = P.layer_mode && !P.token_ids;
  const uint32_t arm = __ldcg(P.status + 1);  // non-zero: timeout test of the router wait
  const int lsh = P.Is > 0 ? 0 : 1;           // first expert slot in use

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
      S.redcnt[s] = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.hfull[i], 1);
      mbar_init(&S.hfree[i], kFW);
    }
    S.ready = 0;
    S.abort_ = 0;
    S.nh = 0;
    S.nhl = 0;
    const int e0 = int((int64_t(P.E) * b) / G), e1 = int((int64_t(P.E) * (b + 1)) / G);
    S.e0 = e0;
    S.ng = P.layer_mode ? e1 - e0 : 0;
    S.w = work_split(P.Is, P.H, P.I, G, 0, b);  // the shared ranges; the rest follow the tables
    S.npos_pre = (S.ng > 0 ? 1 : 0) + (S.w.a.hi - S.w.a.lo);
    S.npos = S.npos_pre;
    fence_mbar_init();
  }
  // the bias before any copy is issued: a global load waits behind the SM's
  // bulk copies in flight
  if (warp == kCtl && learned)
    for (int i = lane; i < P.E; i += 32) sbias[i] = __ldg(P.bias + i);
  __syncthreads();

  if (warp == kProd) {
    // ------------------------------------------------------------ producer
    int issued = 0;
    for (int p = 0;; ++p) {
      if (p >= S.npos_pre && !wait_ready(S)) break;
      if (p >= *reinterpret_cast<volatile int*>(&S.npos) || aborted(S)) break;
      const int s = p % NS;
      if (p >= NS && !fwait(S, &S.empty[s], uint32_t((p / NS) - 1) & 1u, P)) break;
      const FItem m = item_at(P, S, p);
      if (lane == 0) issue_item(P, S, ring + size_t(s) * P.slot_bytes, s, m);
      __syncwarp();
      issued = p + 1;
    }
    // nothing may land in shared memory after the CTA exits: wait for every
    // copy issued (copies complete even after an abort)
    if (lane == 0)
      for (int p = max(0, issued - NS); p < issued; ++p)
        mbar_wait_bounded(&S.full[p % NS], uint32_t(p / NS) & 1u, kWaitTries);
  } else if (warp == kCtl) {
    // ------------------------------------------------------------ control
    bool ok = true;
    if (P.layer_mode) {
      if (S.ng == 0 && lane == 0) atomicAdd(P.ctl + fRoute, 1u);  // nothing to score
      const uint32_t target = uint32_t(G) + (arm ? 1u : 0u);
      ok = fpoll(S, P.ctl + fRoute, target, arm ? arm : kPollTries, P);
      if (ok) {
        for (int i = lane; i < T * P.E; i += 32) ssc[i] = __ldcg(P.scores + i);
        __syncwarp();
        for (int t = 0; t < T; ++t) {
          if (P.token_ids)
            select_hash_warp<true>(t, P.E, P.k, P.vocab, P.routed_scale, ssc + size_t(t) * P.E, P.token_ids,
                                   P.tid2eid, S.sel_ids, S.sel_w, P.status);
          else if (P.E <= 256)
            select_learned_n<false, 8>(t, P.E, P.k, P.routed_scale, ssc + size_t(t) * P.E, sbias, S.sel_ids,
                                       S.sel_w);
          else
            select_learned_n<false, 32>(t, P.E, P.k, P.routed_scale, ssc + size_t(t) * P.E, sbias, S.sel_ids,
                                        S.sel_w);
        }
        __syncwarp();
      }
    } else {
      for (int i = lane; i < T * P.k; i += 32) {
        S.sel_ids[i] = P.topk_ids[i];
        S.sel_w[i] = P.topk_w[i];
      }
      __syncwarp();
    }
    if (ok) {
      build_tables(S, P, P.layer_mode || b != 0);
      if (lane == 0) {
        S.w = work_split(P.Is, P.H, P.I, G, S.nh, b);
        const Work& w = S.w;
        S.npos = S.npos_pre + (w.bq.hi - w.bq.lo) + (w.c.hi - w.c.lo) + (w.d.hi - w.d.lo);
        // the experts whose intermediates this CTA's w2 units read, in item order
        int n = 0;
        if (w.c.hi > w.c.lo) S.hl[n++] = 0;
        if (w.d.hi > w.d.lo) {
          const int per = P.H / 32;
          for (int l = 1 + w.d.lo / per; l <= 1 + (w.d.hi - 1) / per && n < kMaxHSlots; ++l) S.hl[n++] = l;
        }
        S.nhl = n;
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&S.ready) = 1;
      }
      __syncwarp();
      if (b == 0 && P.layer_mode) {
        for (int i = lane; i < T * P.k; i += 32) {
          P.topk_ids[i] = S.sel_ids[i];
          P.topk_w[i] = S.sel_w[i];
        }
        write_perm(S, P);
      }
      // intermediates of the w2 units' experts, into the two staging buffers
      // in turn, once every w13 slab of the expert is done
      const int KM = max(P.I, P.Is);
      int nis = 0;
      for (int j = 0; j < S.nhl && ok; ++j) {
        const int l = S.hl[j], buf = j & 1;
        if (j >= 2) ok = fwait(S, &S.hfree[buf], uint32_t((j >> 1) - 1) & 1u, P);
        const uint32_t need = l == 0 ? uint32_t(P.Is / 4) : uint32_t(P.I / 8);
        ok = ok && fpoll(S, P.ctl + fH + l, need, kPollTries, P);
        if (ok && lane == 0) {
          const int K = l == 0 ? P.Is : P.I;
          mbar_arrive_expect_tx(&S.hfull[buf], uint32_t(T * K * 2));
          // token rows of the expert slot (each KM long), K valid each
          for (int tt = 0; tt < T; ++tt)
            bulk_g2s(hbufs + size_t(buf) * P.hbuf_bytes + size_t(tt) * K * 2, P.dh + (size_t(l) * T + tt) * KM,
                     uint32_t(K * 2), &S.hfull[buf]);
        }
        __syncwarp();
        if (ok) nis = j + 1;
      }
      // copies in flight must land before the CTA exits
      if (lane == 0)
        for (int j = max(0, nis - 2); j < nis; ++j)
          mbar_wait_bounded(&S.hfull[j & 1], uint32_t(j >> 1) & 1u, kWaitTries);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int wi = warp;
    const int g = lane >> 2, t = lane & 3;
    const int nkbH = H / 128;
    // x fragments of the warp's K blocks (wi, wi + 16) into shared memory as
    // f16 scaled by 2^sigma (the token's maximum lands in [2^14, 2^15)):
    // token g's elements kb * 128 + 32 t .. + 31 at xf + ((kb * 4 + t) * T + g) * 64
    {
      uint32_t X[2][16];
      uint32_t mx = 0u;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int kb = wi + 16 * j;
        if (kb < nkbH && g < T) {
          const uint4* src = reinterpret_cast<const uint4*>(P.x + size_t(g) * H + kb * 128 + 32 * t);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(src + q);
            X[j][4 * q] = v.x;
            X[j][4 * q + 1] = v.y;
            X[j][4 * q + 2] = v.z;
            X[j][4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) X[j][i] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = max(mx, max(X[j][i] & 0x7FFFu, (X[j][i] >> 16) & 0x7FFFu));
      }
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (t == 0) S.xmax[wi][g] = mx;
      named_bar_sync(1, kFW * 32);
      uint32_t rmx = 0u;
      for (int w = 0; w < kFW; ++w) rmx = max(rmx, S.xmax[w][g]);
      int sg = 0;
      if (rmx != 0u) {
        const int ef = int(rmx >> 7);
        sg = ef == 0 ? 120 : 141 - ef;  // 14 - floor(log2 max)
        sg = max(-120, min(120, sg));
      }
      if (wi == 0 && t == 0) S.sigma[g] = sg;
      const float mul = __int_as_float((sg + 127) << 23);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int kb = wi + 16 * j;
        if (kb < nkbH && g < T) {
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __half2 hv = __floats2half2_rn(bf16_lo(X[j][i]) * mul, bf16_hi(X[j][i]) * mul);
            h[i] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          uint4* dst = reinterpret_cast<uint4*>(xf + (size_t(kb * 4 + t) * T + g) * 64);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
      }
      named_bar_sync(1, kFW * 32);  // sigma and the fragments visible to every consumer
    }
    const char* xrow = g < T ? xf + (size_t(t) * T + g) * 64 : nullptr;  // K block kb at + kb * 256 * T
    auto bx = [&](int kb) -> const char* { return xrow ? xrow + size_t(kb) * 256 * T : nullptr; };
    int bh_j = -1;               // staging index of the current w2 unit's expert
    const char* hrow = nullptr;  // token g's intermediates in that staging buffer
    auto bhs = [&](int kb) -> const char* { return hrow ? hrow + (kb * 128 + 32 * t) * 2 : nullptr; };
    bool ok = true;
    for (int p = 0;; ++p) {
      if (p >= S.npos_pre && !wait_ready(S)) break;
      if (p >= *reinterpret_cast<volatile int*>(&S.npos) || aborted(S)) break;
      const FItem m = item_at(P, S, p);
      const int s = p % NS;
      if (m.kind == iS2 || m.kind == iR2) {
        const int l = m.kind == iS2 ? 0 : m.l;
        int j = bh_j < 0 ? 0 : bh_j;
        while (j < S.nhl && S.hl[j] != l) ++j;
        if (j != bh_j) {
          // done with the previous expert's buffer; wait for this one's
          if (bh_j >= 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.hfree[bh_j & 1]);
          }
          ok = j < S.nhl && __all_sync(0xffffffffu, fwait(S, &S.hfull[j & 1], uint32_t(j >> 1) & 1u, P));
          if (!ok) break;
          const int K = l == 0 ? P.Is : P.I;
          hrow = g < T ? hbufs + size_t(j & 1) * P.hbuf_bytes + size_t(g) * K * 2 : nullptr;
          bh_j = j;
        }
      }
      ok = __all_sync(0xffffffffu, fwait(S, &S.full[s], uint32_t(p / NS) & 1u, P));
      if (!ok) break;
      const char* st = ring + size_t(s) * P.slot_bytes;
      float4* part = parts + size_t(s) * kFW * 8 * tq;
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      float4 p0 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m.kind == iGate) {
        // router dot products of token g with the CTA's gate rows over the
        // warp's K blocks (x as f16 times 2^sigma)
        float acc[kMaxGateRows];
#pragma unroll
        for (int r = 0; r < kMaxGateRows; ++r) acc[r] = 0.f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int kb = wi + 16 * j;
          if (kb < nkbH) {
            uint32_t B[16];
            load_b(bx(kb), B);
#pragma unroll
            for (int r = 0; r < kMaxGateRows; ++r)
              if (r < S.ng) {
                const uint4* gr = reinterpret_cast<const uint4*>(st + (size_t(r) * H + kb * 128 + 32 * t) * 2);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint4 gv = gr[q];
                  const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    const float2 xv = __half22float2(*reinterpret_cast<const __half2*>(&B[4 * q + i]));
                    acc[r] = fmaf(bf16_lo(gw[i]), xv.x, acc[r]);
                    acc[r] = fmaf(bf16_hi(gw[i]), xv.y, acc[r]);
                  }
                }
              }
          }
        }
#pragma unroll
        for (int r = 0; r < kMaxGateRows; ++r) {
          float a = acc[r];
          a += __shfl_xor_sync(0xffffffffu, a, 1);
          a += __shfl_xor_sync(0xffffffffu, a, 2);
          if (t == 0 && r < S.ng) S.gp[wi][r * 8 + g] = a;
        }
      } else if (m.kind == iR13) {
        const uint8_t* sc = reinterpret_cast<const uint8_t*>(st + 16 * (H / 2));
        float fa, fb;
        ftile_mx<2, 16>(st + g * (H / 2), st + (g + 8) * (H / 2), sc + g * (H / 32), sc + (g + 8) * (H / 32), wi,
                        nkbH, bx, a0, a1, fa, fb);
        p0 = make_float4((a0[0] + a1[0]) * fa, (a0[1] + a1[1]) * fa, (a0[2] + a1[2]) * fb, (a0[3] + a1[3]) * fb);
      } else if (m.kind == iS13) {
        // rows g < 4: gate row g (tile row g) and up row g (tile row g + 8)
        ftile_s8<2, 16>(st + (g & 3) * H, st + (4 + (g & 3)) * H, g < 4, wi, nkbH, bx, a0, a1);
        p0 = make_float4(a0[0] + a1[0], a0[1] + a1[1], a0[2] + a1[2], a0[3] + a1[3]);
      } else if (m.kind == iS2) {
        // shared w2 unit: warp wi owns K block wi
        ftile_s8<1, 16>(st + g * P.Is, st + (g + 8) * P.Is, true, wi, P.Is / 128, bhs, a0, a1);
        p0 = make_float4(a0[0] + a1[0], a0[1] + a1[1], a0[2] + a1[2], a0[3] + a1[3]);
      } else {
        // routed w2 unit: warps 0-7 rows 0-15, warps 8-15 rows 16-31; warp
        // wi owns K blocks wi % 8 and wi % 8 + 8
        const int rs = P.I / 2, Gs = P.I / 32, r0 = 16 * (wi >> 3);
        const uint8_t* sc = reinterpret_cast<const uint8_t*>(st + 32 * rs);
        float fa, fb;
        ftile_mx<2, 8>(st + (r0 + g) * rs, st + (r0 + g + 8) * rs, sc + (r0 + g) * Gs, sc + (r0 + g + 8) * Gs,
                       wi & 7, P.I / 128, bhs, a0, a1, fa, fb);
        p0 = make_float4((a0[0] + a1[0]) * fa, (a0[1] + a1[1]) * fa, (a0[2] + a1[2]) * fb, (a0[3] + a1[3]) * fb);
      }
      if (m.kind != iGate && t < tq) part[(wi * 8 + g) * tq + t] = p0;
      __threadfence_block();
      __syncwarp();
      int old = 0;
      if (lane == 0) old = atomicAdd(&S.redcnt[s], 1);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old != kFW - 1) continue;
      // ---- epilogue: the last warp to post
      __threadfence_block();
      if (lane == 0) S.redcnt[s] = 0;
      epilogue(P, S, m, st, part, s, tq, lsh);
    }
    // a consumer that stops early (abort) must not leave the others waiting
    if (!ok) set_abort(S, P);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(P.ctl + fExit, 1u);
    if (old == uint32_t(G) - 1u) {
      // every CTA is past its waits: reset the counters for the next call
      P.ctl[fRoute] = 0u;
      for (int i = 0; i < kFMaxHit + 1; ++i) P.ctl[fH + i] = 0u;
      for (int i = 0; i < H / 16; ++i) P.ctl[fBlk + i] = 0u;
      __threadfence();
      P.ctl[fExit] = 0u;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------- host side

struct FPlan {
  int nslots = 0, slot_bytes = 0, hbuf_bytes = 0;
  size_t smem = 0;
  bool ok = false;
};

FPlan fplan(const v4moe_config& c, int T, int G) {
  FPlan p;
  const int H = c.hidden, I = c.inter, Is = c.shared_inter, E = c.n_experts;
  if (T < 1 || T > 8 || T * c.top_k > kFMaxHit) return p;
  if (H > 2 * kFW * 128 || I > 16 * 128 || Is > 16 * 128 || H / 16 > 256) return p;
  const int ng = (E + G - 1) / G;
  if (ng > kMaxGateRows) return p;
  uint32_t sb = std::max(bytes_r13(H), bytes_r2(I));
  sb = std::max(sb, uint32_t(ng * H * 2));
  if (Is > 0) sb = std::max(sb, std::max(bytes_s13(H), bytes_s2(Is)));
  p.slot_bytes = int((sb + 127) / 128 * 128);
  p.hbuf_bytes = int((size_t(T) * std::max(I, Is) * 2 + 127) / 128 * 128);
  const int tq = (T + 1) / 2;
  const size_t fixed = kFHead + size_t(T) * H * 2 + 2 * size_t(p.hbuf_bytes) + size_t(T) * E * 4 + size_t(E) * 4 + 128;
  const size_t per_slot = size_t(p.slot_bytes) + size_t(kFW) * 8 * tq * 16;
  const size_t room = 227 * 1024;
  if (fixed + 2 * per_slot > room) return p;
  p.nslots = int(std::min<size_t>(kMaxSlots, (room - fixed) / per_slot));
  p.smem = fixed + p.nslots * per_slot;
  p.ok = true;
  return p;
}

// 2^floor(log2(f16 max / bound)) for intermediates bounded by `bound`.
float h_scale(float bound) {
  int e = 0;
  while (e < 14 && bound * std::ldexp(1.0f, e + 1) < 65504.0f) ++e;
  return std::ldexp(1.0f, e);
}

}  // namespace

DecodeBuffers dec_buffers(const v4moe_config& c, int64_t T) {
  DecodeBuffers b;
  if (T < 1 || T > kDecodeMaxTokens) return b;
  b.ctl = size_t(fWords) * 4;
  b.dh = size_t(kFMaxHit + 1) * T * std::max(c.inter, c.shared_inter) * 2;
  b.part = size_t(kFMaxHit + 1) * c.hidden * T * 4;
  return b;
}

// The shared expert's fp32 row scales travel by bulk copy (16-byte aligned).
bool dec_supported(const v4moe_config& c, int T, const v4moe_weights& w) {
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (c.shared_inter > 0 && (!a16(w.sh_w13_scale) || !a16(w.sh_w2_scale))) return false;
  return fplan(c, T, device_sms()).ok;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  const v4moe_config& c = a.c;
  const int G = device_sms();
  const FPlan pl = fplan(c, a.T, G);
  if (!pl.ok) return cudaErrorInvalidValue;
  FParams P;
  P.T = a.T;
  P.H = c.hidden;
  P.I = c.inter;
  P.Is = c.shared_inter;
  P.E = c.n_experts;
  P.k = c.top_k;
  P.vocab = c.vocab;
  P.limit = c.swiglu_limit;
  P.routed_scale = c.routed_scale;
  // |h| <= L * L * routed_scale (routed, weights <= routed_scale), L * L (shared)
  const float L = c.swiglu_limit;
  P.tau_r = h_scale(L * L * std::max(1.0f, std::fabs(c.routed_scale)));
  P.tau_s = h_scale(L * L);
  P.layer_mode = a.layer_mode;
  P.nslots = pl.nslots;
  P.slot_bytes = pl.slot_bytes;
  P.hbuf_bytes = pl.hbuf_bytes;
  P.G = G;
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
  P.scores = a.scores;
  P.w13_codes = a.w.w13_codes;
  P.w13_scales = a.w.w13_scales;
  P.w2_codes = a.w.w2_codes;
  P.w2_scales = a.w.w2_scales;
  P.sh13 = a.w.sh_w13;
  P.sh13_scale = a.w.sh_w13_scale;
  P.sh2 = a.w.sh_w2;
  P.sh2_scale = a.w.sh_w2_scale;
  P.dh = a.dh;
  P.part = a.part;
  P.ctl = a.ctl;
  P.status = a.status;
  P.out = a.out;
  set_smem(k_dec_fused, pl.smem);
  return launch_kernel("dec_fused", k_dec_fused, dim3(G), dim3(kFThreads), pl.smem, st, false, P);
}

}  // namespace v4moe
