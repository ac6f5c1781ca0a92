// C-ABI entry points of libv4moe: argument validation, workspace carve-up and
// dispatch to the kernels. The declarations and their contracts are in
// include/v4moe.h.
#include <cudaTypedefs.h>

#include <mutex>
#include <unordered_map>

#include "v4moe_internal.cuh"

namespace v4moe {

bool config_ok(const v4moe_config* c) {
  if (!c) return false;
  if (c->hidden <= 0 || c->hidden % 128 != 0) return false;
  if (c->inter <= 0 || c->inter % 128 != 0) return false;
  if (c->shared_inter < 0 || c->shared_inter % 128 != 0) return false;
  if (c->top_k < 1 || c->top_k > 8) return false;
  if (c->n_experts < c->top_k || c->n_experts > 1024) return false;
  if (!(c->routed_scale == c->routed_scale) || !(c->swiglu_limit > 0.0f)) return false;
  return true;
}

namespace {
struct DevInfo {
  bool ok = false;
  int sms = 0;
};
std::mutex g_dev_mu;
std::unordered_map<int, DevInfo> g_dev;

// The current device's cached attributes (queried once per device).
const DevInfo* device_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  auto it = g_dev.find(dev);
  if (it == g_dev.end()) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    DevInfo d;
    d.ok = major == 10 && minor == 0;
    d.sms = sms;
    it = g_dev.emplace(dev, d).first;
  }
  return &it->second;
}
}  // namespace

int32_t check_device() {
  const DevInfo* d = device_info();
  return d && d->ok ? V4MOE_OK : V4MOE_ERR_UNSUPPORTED_DEVICE;
}

int device_sms() {
  const DevInfo* d = device_info();
  return d && d->sms > 0 ? d->sms : 148;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_tensor_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  const auto fn = tensor_map_encoder();
  if (!fn || rank < 2 || rank > 3) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  return fn(m, dt, cuuint32_t(rank), const_cast<void*>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int32_t check_ws(const v4moe_config* c, int32_t T, const void* ws, size_t ws_bytes) {
  if (!ws || !aligned(ws, 256)) return V4MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(*c, T).total) return V4MOE_ERR_WORKSPACE;
  return V4MOE_OK;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int32_t launch_status(cudaError_t e) {
  if (e != cudaSuccess) {
    cudaGetLastError();
    return V4MOE_ERR_LAUNCH;
  }
  return V4MOE_OK;
}

}  // namespace
}  // namespace v4moe

using namespace v4moe;

extern "C" {

size_t v4moe_workspace_bytes(const v4moe_config* cfg, int32_t T) {
  if (!config_ok(cfg) || T < 0) return 0;
  return ws_layout(*cfg, T).total;
}

int32_t v4moe_route(const v4moe_config* cfg, int32_t T, const void* x, const void* gate,
                    const float* bias, const int32_t* token_ids, const int32_t* tid2eid,
                    int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  if (!config_ok(cfg) || T < 0) return V4MOE_ERR_INVALID_ARG;
  const bool hash = token_ids != nullptr || tid2eid != nullptr;
  if (hash && (bias || !token_ids || !tid2eid || cfg->vocab <= 0)) return V4MOE_ERR_INVALID_ARG;
  if (!hash && !bias) return V4MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (!x || !gate || !topk_ids || !topk_w) return V4MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(gate, 16) || !aligned(topk_ids, 4) || !aligned(topk_w, 4))
      return V4MOE_ERR_INVALID_ARG;
  }
  if (int32_t r = check_ws(cfg, T, ws, ws_bytes)) return r;
  if (int32_t r = check_device()) return r;
  if (T == 0) return V4MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  return launch_status(launch_route(*cfg, T, static_cast<const __nv_bfloat16*>(x),
                                    static_cast<const __nv_bfloat16*>(gate), bias, token_ids, tid2eid,
                                    topk_ids, topk_w, at<float>(ws, L.scores), at<uint32_t>(ws, L.status),
                                    static_cast<cudaStream_t>(stream)));
}

int32_t v4moe_permute(const v4moe_config* cfg, int32_t T, const int32_t* topk_ids, int32_t* counts,
                      int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos, void* ws,
                      size_t ws_bytes, void* stream) {
  if (!config_ok(cfg) || T < 0) return V4MOE_ERR_INVALID_ARG;
  if (!counts || !offsets) return V4MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !sorted_slot || !slot_pos)) return V4MOE_ERR_INVALID_ARG;
  if (int64_t(T) * cfg->top_k > 0x7fffffff / 2) return V4MOE_ERR_INVALID_ARG;
  if (int32_t r = check_ws(cfg, T, ws, ws_bytes)) return r;
  if (int32_t r = check_device()) return r;
  const WsLayout L = ws_layout(*cfg, T);
  return launch_status(launch_permute(*cfg, T, topk_ids, counts, offsets, sorted_slot, slot_pos,
                                      at<int32_t>(ws, L.chunk_counts), at<int32_t>(ws, L.chunk_base),
                                      L.nchunks, at<uint32_t>(ws, L.status),
                                      static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace v4moe {
namespace {

int32_t check_weights(const v4moe_config* cfg, const v4moe_weights* weights) {
  if (!weights) return V4MOE_ERR_INVALID_ARG;
  const v4moe_weights& w = *weights;
  if (!w.w13_codes || !w.w13_scales || !w.w2_codes || !w.w2_scales) return V4MOE_ERR_INVALID_ARG;
  if (!aligned(w.w13_codes, 16) || !aligned(w.w2_codes, 16) || !aligned(w.w13_scales, 16) ||
      !aligned(w.w2_scales, 16))
    return V4MOE_ERR_INVALID_ARG;
  if (cfg->shared_inter > 0) {
    if (!w.sh_w13 || !w.sh_w13_scale || !w.sh_w2 || !w.sh_w2_scale) return V4MOE_ERR_INVALID_ARG;
    if (!aligned(w.sh_w13, 16) || !aligned(w.sh_w2, 16) || !aligned(w.sh_w13_scale, 4) ||
        !aligned(w.sh_w2_scale, 4))
      return V4MOE_ERR_INVALID_ARG;
  }
  return V4MOE_OK;
}

ForwardArgs forward_args(const v4moe_config* cfg, int32_t T, const void* x, const int32_t* topk_ids,
                         const float* topk_w, const int32_t* offsets, const int32_t* sorted_slot,
                         const int32_t* slot_pos, const v4moe_weights* weights, void* out, void* ws) {
  const WsLayout L = ws_layout(*cfg, T);
  ForwardArgs a;
  a.c = *cfg;
  a.T = T;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.topk_ids = topk_ids;
  a.topk_w = topk_w;
  a.offsets = offsets;
  a.sorted_slot = sorted_slot;
  a.slot_pos = slot_pos;
  a.w = *weights;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.status = at<uint32_t>(ws, L.status);
  a.h = at<__nv_bfloat16>(ws, L.h);
  a.y_slot = at<__nv_bfloat16>(ws, L.y_slot);
  a.hs = at<__nv_bfloat16>(ws, L.hs);
  a.ys = at<float>(ws, L.ys);
  return a;
}

// Arguments of the single-kernel decode path; routing pointers are filled in
// by the caller for layer mode.
DecodeArgs decode_args(const v4moe_config* cfg, int32_t T, const void* x, const v4moe_weights* weights, void* out,
                       void* ws) {
  const WsLayout L = ws_layout(*cfg, T);
  DecodeArgs d = {};
  d.c = *cfg;
  d.T = T;
  d.x = static_cast<const __nv_bfloat16*>(x);
  d.w = *weights;
  d.out = static_cast<__nv_bfloat16*>(out);
  d.status = at<uint32_t>(ws, L.status);
  d.ctl = at<uint32_t>(ws, L.d_ctl);
  d.dh = at<__half>(ws, L.d_dh);
  d.hs = at<__half>(ws, L.d_hs);
  return d;
}

}  // namespace
}  // namespace v4moe

extern "C" {

int32_t v4moe_forward(const v4moe_config* cfg, int32_t T, const void* x, const int32_t* topk_ids,
                      const float* topk_w, const int32_t* offsets, const int32_t* sorted_slot,
                      const int32_t* slot_pos, const v4moe_weights* weights, void* out, void* ws,
                      size_t ws_bytes, void* stream) {
  if (!config_ok(cfg) || T < 0) return V4MOE_ERR_INVALID_ARG;
  if (int32_t r = check_weights(cfg, weights)) return r;
  if (!offsets) return V4MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (!x || !topk_ids || !topk_w || !sorted_slot || !slot_pos || !out) return V4MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16)) return V4MOE_ERR_INVALID_ARG;
    if (x == out) return V4MOE_ERR_INVALID_ARG;
  }
  if (int32_t r = check_ws(cfg, T, ws, ws_bytes)) return r;
  if (int32_t r = check_device()) return r;
  if (T == 0) return V4MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dec_supported(*cfg, T)) {
    DecodeArgs d = decode_args(cfg, T, x, weights, out, ws);
    d.layer_mode = 0;
    d.topk_ids = const_cast<int32_t*>(topk_ids);
    d.topk_w = const_cast<float*>(topk_w);
    return launch_status(launch_decode(d, st));
  }
  const ForwardArgs a = forward_args(cfg, T, x, topk_ids, topk_w, offsets, sorted_slot, slot_pos, weights, out, ws);
  return launch_status(
      launch_forward_tc(a, at<__half>(ws, L.xlog), at<int>(ws, L.sigma), at<char>(ws, L.tc), at<char>(ws, L.sh16), st));
}

int32_t v4moe_layer(const v4moe_config* cfg, int32_t T, const void* x, const void* gate, const float* bias,
                    const int32_t* token_ids, const int32_t* tid2eid, const v4moe_weights* weights,
                    int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets, int32_t* sorted_slot,
                    int32_t* slot_pos, void* out, void* ws, size_t ws_bytes, void* stream) {
  if (!config_ok(cfg) || T < 0) return V4MOE_ERR_INVALID_ARG;
  if (int32_t r = check_weights(cfg, weights)) return r;
  const bool hash = token_ids != nullptr || tid2eid != nullptr;
  if (hash && (bias || !token_ids || !tid2eid || cfg->vocab <= 0)) return V4MOE_ERR_INVALID_ARG;
  if (!hash && !bias) return V4MOE_ERR_INVALID_ARG;
  if (!counts || !offsets) return V4MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (!x || !gate || !topk_ids || !topk_w || !sorted_slot || !slot_pos || !out) return V4MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(gate, 16) || !aligned(out, 16) || x == out) return V4MOE_ERR_INVALID_ARG;
  }
  if (int64_t(T) * cfg->top_k > 0x7fffffff / 2) return V4MOE_ERR_INVALID_ARG;
  if (int32_t r = check_ws(cfg, T, ws, ws_bytes)) return r;
  if (int32_t r = check_device()) return r;
  // an empty batch still reports empty counts and offsets
  if (T == 0) return v4moe_permute(cfg, 0, topk_ids, counts, offsets, sorted_slot, slot_pos, ws, ws_bytes, stream);
  if (dec_supported(*cfg, T)) {
    DecodeArgs d = decode_args(cfg, T, x, weights, out, ws);
    d.layer_mode = 1;
    d.gate = static_cast<const __nv_bfloat16*>(gate);
    d.bias = bias;
    d.token_ids = token_ids;
    d.tid2eid = tid2eid;
    d.topk_ids = topk_ids;
    d.topk_w = topk_w;
    d.counts = counts;
    d.offsets = offsets;
    d.sorted_slot = sorted_slot;
    d.slot_pos = slot_pos;
    return launch_status(launch_decode(d, static_cast<cudaStream_t>(stream)));
  }
  if (int32_t r = v4moe_route(cfg, T, x, gate, bias, token_ids, tid2eid, topk_ids, topk_w, ws, ws_bytes, stream))
    return r;
  if (int32_t r = v4moe_permute(cfg, T, topk_ids, counts, offsets, sorted_slot, slot_pos, ws, ws_bytes, stream))
    return r;
  return v4moe_forward(cfg, T, x, topk_ids, topk_w, offsets, sorted_slot, slot_pos, weights, out, ws, ws_bytes,
                       stream);
}

size_t v4moe_linear_w8a16_grouped_workspace_bytes(int32_t T, int32_t G, int32_t N, int32_t K) {
  if (T < 0 || G <= 0 || N <= 0 || K <= 0) return 0;
  return linear_w8a16_ws_bytes(G, N, K);
}

int32_t v4moe_linear_w8a16_grouped(int32_t T, int32_t G, int32_t N, int32_t K, const void* x, const int8_t* q,
                                   const float* scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || G <= 0 || N <= 0 || K <= 0 || N % 32 != 0 || K % 64 != 0) return V4MOE_ERR_INVALID_ARG;
  if (int64_t(G) * N > (int64_t(1) << 30) || int64_t(G) * K > (int64_t(1) << 30)) return V4MOE_ERR_INVALID_ARG;
  if (!q || !scale || !aligned(q, 16) || !aligned(scale, 4)) return V4MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out || !aligned(x, 16) || !aligned(out, 16) || x == out)) return V4MOE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return V4MOE_ERR_INVALID_ARG;
  if (ws_bytes < linear_w8a16_ws_bytes(G, N, K)) return V4MOE_ERR_WORKSPACE;
  if (int32_t r = check_device()) return r;
  if (T == 0) return V4MOE_OK;
  return launch_status(launch_linear_w8a16(T, G, N, K, static_cast<const __nv_bfloat16*>(x), q, scale,
                                           static_cast<__nv_bfloat16*>(out), static_cast<char*>(ws),
                                           static_cast<cudaStream_t>(stream)));
}

size_t v4moe_linear_w8a16_workspace_bytes(int32_t T, int32_t N, int32_t K) {
  return v4moe_linear_w8a16_grouped_workspace_bytes(T, 1, N, K);
}

int32_t v4moe_linear_w8a16(int32_t T, int32_t N, int32_t K, const void* x, const int8_t* q, const float* scale,
                           void* out, void* ws, size_t ws_bytes, void* stream) {
  return v4moe_linear_w8a16_grouped(T, 1, N, K, x, q, scale, out, ws, ws_bytes, stream);
}

int32_t v4moe_read_device_status(const void* ws, void* stream) {
  if (!ws || !aligned(ws, 256)) return V4MOE_ERR_INVALID_ARG;
  uint32_t word = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return V4MOE_ERR_LAUNCH;
  }
  if (word & kStatusTimeout) return V4MOE_ERR_TIMEOUT;
  if (word & (kStatusBadExpertId | kStatusBadTokenId)) return V4MOE_ERR_DATA;
  return V4MOE_OK;
}

int32_t v4moe_clear_device_status(void* ws, void* stream) {
  if (!ws || !aligned(ws, 256)) return V4MOE_ERR_INVALID_ARG;
  return launch_status(cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)));
}

const char* v4moe_status_string(int32_t s) {
  switch (s) {
    case V4MOE_OK: return "ok";
    case V4MOE_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer or bad shape)";
    case V4MOE_ERR_WORKSPACE: return "workspace too small";
    case V4MOE_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0)";
    case V4MOE_ERR_LAUNCH: return "kernel launch failed";
    case V4MOE_ERR_DATA: return "device flagged out-of-range expert or token ids";
    case V4MOE_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    default: return "unknown status";
  }
}

}  // extern "C"
