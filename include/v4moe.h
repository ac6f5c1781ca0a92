/*
 * libv4moe — routed Mixture-of-Experts FFN layer of DeepSeek-V4-Flash on one
 * NVIDIA B200 (sm_100a).
 *
 * The layer (sources: "appmana/deepseek-v4-mxfp4-int8 config.json",
 * quantization_config and MoE keys; "DeepSeek-V4-Flash-0731" catalog page,
 * table "Checked in its code", rows "Mixture of experts", "Shared expert",
 * "Auxiliary-loss-free load balancing (selection bias)", "SwiGLU
 * feed-forward"; "DeepSeek-V4-Flash export design", section "Source
 * configuration"):
 *
 *   s      = sqrt(softplus(x . gate^T))                      [T, E]
 *   ids    = top-k(s + bias)   or   tid2eid[token_id]         [T, k]
 *   w      = routed_scale * s[ids] / sum(s[ids])              [T, k]
 *   out[t] = sum_j w[t,j] * FFN_{ids[t,j]}(x[t]) + FFN_shared(x[t])
 *   FFN(x) = W2 * (silu(min(g, L)) * clamp(u, -L, L)),  [g; u] = W13 * x
 *
 * Routed W13 [2I, H] / W2 [H, I] are MXFP4: E2M1 codes, two per byte along K
 * (even K index in the low nibble), one E8M0 scale byte per 32 K elements.
 * The shared expert's W13 / W2 are int8, symmetric, one fp32 scale per output
 * row. Activations are bf16; accumulation is fp32.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller, row-major and
 *    contiguous, 16-byte aligned unless stated otherwise. bf16 tensors are
 *    passed as void* (2-byte elements, IEEE bfloat16).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *    asynchronous on it; none synchronises, allocates device memory or reads
 *    device memory on the host, except v4moe_read_device_status (which
 *    synchronises the stream, for tests and debugging).
 *  - Scratch memory comes from the caller's workspace `ws` of `ws_bytes`
 *    bytes (see v4moe_workspace_bytes); it must be 256-byte aligned and
 *    zero-filled before its first use (every call leaves its first 256 bytes
 *    in a state the next call accepts; v4moe_clear_device_status restores
 *    them). Those bytes hold a device status word that kernels set when they
 *    meet bad data (an out-of-range expert or token id, which they skip) or
 *    give up a bounded wait; read it with v4moe_read_device_status. Word 1
 *    of the block is a test hook of the decode path (T <= 8): when non-zero,
 *    the expert kernel first waits on a barrier that nothing arrives at,
 *    gives up after that many polls (status V4MOE_ERR_TIMEOUT) and returns
 *    without computing; zero (the default, and what
 *    v4moe_clear_device_status writes) disarms it. Calls that share a
 *    workspace must not overlap on the GPU.
 *  - Return value: a V4MOE_* status code. Argument errors are detected on the
 *    host before anything is launched; data errors are visible only through
 *    the device status word.
 *  - The library keeps no state between calls except a per-device cache of
 *    device attributes and kernel attributes (thread-safe).
 */
#ifndef V4MOE_H_
#define V4MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define V4MOE_OK 0
#define V4MOE_ERR_INVALID_ARG 1        /* null/misaligned pointer, bad shape or size */
#define V4MOE_ERR_WORKSPACE 2          /* workspace smaller than v4moe_workspace_bytes */
#define V4MOE_ERR_UNSUPPORTED_DEVICE 3 /* current device is not compute capability 10.0 */
#define V4MOE_ERR_LAUNCH 4             /* a kernel launch failed (cudaGetLastError) */
#define V4MOE_ERR_DATA 5               /* device flagged out-of-range ids (status word) */
#define V4MOE_ERR_TIMEOUT 6            /* a bounded device-side wait gave up (status word) */

/* Layer shape and constants ("config.json": hidden_size, moe_intermediate_size,
 * n_routed_experts, num_experts_per_tok, vocab_size, routed_scaling_factor,
 * swiglu_limit; the shared expert has moe_intermediate_size too).
 * Requirements: hidden % 128 == 0, inter % 128 == 0, shared_inter % 128 == 0
 * (0 = no shared expert), 1 <= top_k <= 8, top_k <= n_experts <= 1024. */
typedef struct v4moe_config {
  int32_t hidden;        /* H: 4096 */
  int32_t inter;         /* I: 2048 */
  int32_t n_experts;     /* E: 256 */
  int32_t top_k;         /* k: 6 */
  int32_t shared_inter;  /* I_s: 2048, or 0 */
  int32_t vocab;         /* rows of tid2eid (hash routing): 129280 */
  float routed_scale;    /* 1.5 */
  float swiglu_limit;    /* 10.0 */
} v4moe_config;

/* Expert weights (device pointers, caller-owned, never written).
 *  w13_codes  [E, 2I, H/2] uint8   rows [0, I) gate (w1), rows [I, 2I) up (w3)
 *  w13_scales [E, 2I, H/32] uint8  E8M0
 *  w2_codes   [E, H, I/2]  uint8
 *  w2_scales  [E, H, I/32] uint8   E8M0
 *  sh_w13     [2I_s, H] int8, sh_w13_scale [2I_s] fp32  (gate rows then up rows)
 *  sh_w2      [H, I_s]  int8, sh_w2_scale  [H] fp32
 * Code pointers and E8M0 scale pointers must be 16-byte aligned, fp32 scale
 * pointers 4-byte aligned. The shared-expert pointers may be NULL only when
 * shared_inter == 0. */
typedef struct v4moe_weights {
  const uint8_t* w13_codes;
  const uint8_t* w13_scales;
  const uint8_t* w2_codes;
  const uint8_t* w2_scales;
  const int8_t* sh_w13;
  const float* sh_w13_scale;
  const int8_t* sh_w2;
  const float* sh_w2_scale;
} v4moe_weights;

/* Bytes of workspace that v4moe_route / v4moe_permute / v4moe_forward need for
 * T tokens (the maximum over the three calls). Returns 0 for an invalid
 * config or T < 0. Pure host function. */
size_t v4moe_workspace_bytes(const v4moe_config* cfg, int32_t T);

/* Router ("Checked in its code" rows "Mixture of experts" and "Auxiliary-loss-
 * free load balancing": top-k of scores + e_score_correction_bias selects,
 * the unbiased scores weight; "config.json" scoring_func sqrtsoftplus,
 * norm_topk_prob true, routed_scaling_factor; hash layers: "DeepSeek-V4-Flash
 * export design", first three layers select experts from a token-id hash
 * table).
 *   x         [T, H] bf16;  gate [E, H] bf16
 *   bias      [E] fp32  -> learned routing (token_ids and tid2eid must be NULL)
 *   token_ids [T] int32 and tid2eid [vocab, k] int32 -> hash routing (bias NULL)
 *   topk_ids  [T, k] int32 out: learned -> the k selected experts in ascending
 *             id (ties in s + bias go to the lower id); hash -> the table row
 *   topk_w    [T, k] fp32 out: routed_scale * s[id] / sum over the k ids
 * Scores are fp32 (bf16 products, fp32 accumulation). An out-of-range token id
 * or table entry sets V4MOE_ERR_DATA in the status word; that token gets
 * expert 0 with weight 0. T == 0 is a no-op. */
int32_t v4moe_route(const v4moe_config* cfg, int32_t T, const void* x, const void* gate,
                    const float* bias, const int32_t* token_ids, const int32_t* tid2eid,
                    int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Token permutation by expert: a stable counting sort of the T*k slots
 * s = t*k + j by topk_ids (the grouping behind experts(flat, indices,
 * weights), "Checked in its code" row "Shared expert").
 *   counts      [E] int32 out: slots per expert
 *   offsets     [E+1] int32 out: exclusive prefix sum of counts
 *   sorted_slot [T*k] int32 out: slots grouped by ascending expert, ascending s
 *               within an expert
 *   slot_pos    [T*k] int32 out: inverse of sorted_slot
 * Out-of-range ids set V4MOE_ERR_DATA and are left out of every output (the
 * arrays are then incomplete). Integer results are deterministic. */
int32_t v4moe_permute(const v4moe_config* cfg, int32_t T, const int32_t* topk_ids,
                      int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                      int32_t* slot_pos, void* ws, size_t ws_bytes, void* stream);

/* v4moe_permute without a workspace, for callers that cannot allocate device
 * memory (the paper has no counterpart: this is a deployment variant).
 * Some runtimes plan all device memory at start-up and forbid allocations
 * afterwards, and some host code must not reach a device allocator at all
 * (it may synchronise the device or fail under memory pressure). This entry
 * point computes exactly what v4moe_permute computes, with the same arguments
 * minus ws/ws_bytes; its scratch is a fixed array of about 256 KiB inside the
 * library that every GPU loading the library holds until the process exits.
 *  - Limits: T * top_k <= 65536 and n_experts <= 1024; larger sizes return
 *    V4MOE_ERR_INVALID_ARG before anything is launched.
 *  - It allocates nothing (no cudaMalloc/cudaFree, no allocating library
 *    call). The first call on a device looks up the array's device address
 *    with cudaGetSymbolAddress (once per device, with that device current)
 *    and keeps it for the life of the process; make that first call before
 *    any stream capture. A device reset (cudaDeviceReset) after that first
 *    call is not supported: the kept address would no longer be valid.
 *  - Every call shares the one array. Calls whose kernels may overlap on the
 *    GPU (different streams, or several host threads) race on it and must be
 *    serialised by the caller.
 *  - Out-of-range ids are skipped as in v4moe_permute, but the device status
 *    word is internal to the array (cleared at the start of each call) and
 *    cannot be read back; use v4moe_permute when errors must be reported. */
int32_t v4moe_permute_static(const v4moe_config* cfg, int32_t T, const int32_t* topk_ids,
                             int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                             int32_t* slot_pos, void* stream);

/* Expert computation and combine:
 *   out[t] = bf16( sum_j topk_w[t,j] * FFN_{topk_ids[t,j]}(x[t]) + FFN_shared(x[t]) )
 * with the clamped SwiGLU ("Checked in its code" row "SwiGLU feed-forward":
 * gate clamped above at swiglu_limit, up clamped on both sides). Routing may
 * come from v4moe_route/v4moe_permute or from the caller (offsets/sorted_slot/
 * slot_pos must be the permutation of topk_ids). x [T, H] bf16, out [T, H] bf16
 * (may not alias x). The intermediate h = swiglu(g, u) enters the down
 * projection with at least 16-bit float precision (W4A16: 16-bit
 * activations): as f16 on the decode and small-batch paths, and on the
 * block-scaled tensor-core path as two E4M3 planes with E8M0 scales per 32
 * channels, which hold an f16-rounded h exactly for values within 2^-14 of
 * their block's largest magnitude (smaller ones keep their leading bits). */
int32_t v4moe_forward(const v4moe_config* cfg, int32_t T, const void* x,
                      const int32_t* topk_ids, const float* topk_w, const int32_t* offsets,
                      const int32_t* sorted_slot, const int32_t* slot_pos,
                      const v4moe_weights* weights, void* out, void* ws, size_t ws_bytes,
                      void* stream);

/* The whole layer in one call: v4moe_route, v4moe_permute and v4moe_forward
 * with the same arguments and results (routing outputs included). For small
 * batches (T <= 8) the router runs as one thread-block cluster (up to 16
 * CTAs) whose leader selects each token's experts and writes the routing
 * outputs and the permutation, and the two expert kernels, chained to it by
 * programmatic dependent launch, start streaming the shared expert's weights
 * before the routing is known. Intermediates on this path are f16 of h
 * times a fixed power of two derived from swiglu_limit (divided out in the
 * down projection). */
int32_t v4moe_layer(const v4moe_config* cfg, int32_t T, const void* x, const void* gate,
                    const float* bias, const int32_t* token_ids, const int32_t* tid2eid,
                    const v4moe_weights* weights, int32_t* topk_ids, float* topk_w,
                    int32_t* counts, int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos,
                    void* out, void* ws, size_t ws_bytes, void* stream);

/* W8A16 linear ("config.json" quantization_config, group "linears_w8a16":
 * int8 weights, symmetric, one scale per output channel, 16-bit float
 * activations; its targets are the attention projections fused_wqa_wkv,
 * wq_b, wo_a, wo_b, the indexer's wq_b and compressor wkv, and the shared
 * expert's gate_up_proj / down_proj):
 *   out[t, n] = bf16( scale[n] * sum_k q[n, k] * x[t, k] ),  fp32 accumulation
 *   x [T, K] bf16, q [N, K] int8 (row-major, 16-byte aligned), scale [N] fp32,
 *   out [T, N] bf16 (16-byte aligned, may not alias x).
 * Requirements: N % 32 == 0, K % 64 == 0. The weights are widened exactly to
 * bf16 in the workspace (v4moe_linear_w8a16_workspace_bytes(T, N, K) bytes,
 * 256-byte aligned; its first 256 bytes hold the device status word as for
 * the other calls) and multiplied on the tensor cores. T == 0 is a no-op. */
size_t v4moe_linear_w8a16_workspace_bytes(int32_t T, int32_t N, int32_t K);
int32_t v4moe_linear_w8a16(int32_t T, int32_t N, int32_t K, const void* x, const int8_t* q,
                           const float* scale, void* out, void* ws, size_t ws_bytes, void* stream);

/* The same linear in G independent groups (the config's wo_a: o_groups = 8
 * groups of heads, each projected by its own o_lora_rank x (heads per group *
 * head_dim) block of one weight matrix):
 *   out[t, g N + n] = bf16( scale[g N + n] * sum_k q[g N + n, k] * x[t, g K + k] )
 *   x [T, G K] bf16, q [G N, K] int8, scale [G N] fp32, out [T, G N] bf16,
 * alignment and requirements as above (N % 32 == 0, K % 64 == 0, G >= 1;
 * G N and G K at most 2^30); workspace
 * v4moe_linear_w8a16_grouped_workspace_bytes(T, G, N, K) bytes. G == 1 is
 * v4moe_linear_w8a16. */
size_t v4moe_linear_w8a16_grouped_workspace_bytes(int32_t T, int32_t G, int32_t N, int32_t K);
int32_t v4moe_linear_w8a16_grouped(int32_t T, int32_t G, int32_t N, int32_t K, const void* x,
                                   const int8_t* q, const float* scale, void* out, void* ws,
                                   size_t ws_bytes, void* stream);

/* Synchronises `stream`, reads the device status word of `ws` and returns
 * V4MOE_OK, V4MOE_ERR_DATA or V4MOE_ERR_TIMEOUT (or V4MOE_ERR_LAUNCH if the
 * copy fails). Test/debug only. */
int32_t v4moe_read_device_status(const void* ws, void* stream);

/* Clears the device status word (asynchronous on stream). */
int32_t v4moe_clear_device_status(void* ws, void* stream);

/* Static description of a status code; never NULL. */
const char* v4moe_status_string(int32_t status);


/* ---- Instrumentation (benchmarks, profiling) ------------------------------
 * No counterpart in the layer's definition: these report what the library
 * launched. Kernel timing is off by default; while it is on, every kernel
 * launch is bracketed by two CUDA events recorded on its stream (which also
 * disables programmatic dependent launch, so use it in a separate pass). */

/* Switch per-kernel event timing on (on != 0) or off. */
int32_t v4moe_profile_enable(int32_t on);

/* Forget the launches timed so far (events are kept for reuse). */
int32_t v4moe_profile_reset(void);

/* Waits for the timed launches and aggregates them per kernel name:
 * names [max_entries][name_len] (NUL-terminated), total_ms and launches per
 * name; *n_entries = number of distinct names (may exceed max_entries). */
int32_t v4moe_profile_read(char* names, int32_t name_len, float* total_ms, int32_t* launches,
                           int32_t max_entries, int32_t* n_entries);

/* Number of kernels the library has launched in this process. */
uint64_t v4moe_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* V4MOE_H_ */
