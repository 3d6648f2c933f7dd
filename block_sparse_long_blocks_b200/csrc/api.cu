// C ABI entry points: argument validation, derived geometry, workspace layout,
// launches on the caller's stream, and the device status word.
#include <cmath>
#include <cstdio>
#include <cstdint>
#include <mutex>

#include "internal.cuh"

namespace fp {

// Device-side error bits (FP_DEV_*); set by kernels, read/cleared by fp_get_device_status.
__device__ unsigned g_device_status;

thread_local char t_last_error[256] = "";

void set_last_error(const char* step, int code, const char* detail) {
  snprintf(t_last_error, sizeof(t_last_error), "%s failed (code %d): %s", step, code, detail ? detail : "");
}

namespace {

constexpr int kMaxDevices = 64;

fp_status_t cuda_fail(const char* step, cudaError_t e) {
  set_last_error(step, (int)e, cudaGetErrorString(e));
  return FP_ERR_CUDA;
}

unsigned* status_ptr() {
  static unsigned* ptrs[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned*>(p);
  }
  return ptrs[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// Validates everything that does not touch the device. `attention` selects the
// attention kernel's extra limits.
fp_status_t validate(const fp_params_t* p, bool attention) {
  if (!p) return FP_ERR_INVALID_ARG;
  if (p->dtype != FP_BF16 && p->dtype != FP_E4M3) return FP_ERR_INVALID_ARG;
  if (p->batch < 1 || p->max_seqlen < 1 || p->hq < 1 || p->hkv < 1 || p->hq % p->hkv != 0)
    return FP_ERR_INVALID_ARG;
  if (!std::isfinite(p->alpha) || p->alpha < 0.f) return FP_ERR_INVALID_ARG;
  if (p->sink_tokens < 0 || p->window_tokens < 0) return FP_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale) || p->softmax_scale < 0.f) return FP_ERR_INVALID_ARG;
  // head dim 128, or 64 with bf16 inputs (an e4m3 row of 64 would be 64 bytes,
  // below the kernels' 128-byte swizzled rows)
  if (p->head_dim != 128 && !(p->head_dim == 64 && p->dtype == FP_BF16)) return FP_ERR_UNSUPPORTED;
  if (p->block != 64 && p->block != 128) return FP_ERR_UNSUPPORTED;
  const int G = p->hq / p->hkv;
  if (!(G <= 8 || G == 16)) return FP_ERR_UNSUPPORTED;
  const long long Nmax = ceil_div(p->max_seqlen, p->block);
  if (Nmax > 8192) return FP_ERR_UNSUPPORTED;
  if (p->dtype == FP_E4M3 && (!p->q_scale || !p->k_scale || (attention && !p->v_scale)))
    return FP_ERR_INVALID_ARG;
  if (p->cu_seqlens) {
    if (p->total_tokens < 0) return FP_ERR_INVALID_ARG;
    if (!aligned(p->cu_seqlens, 4)) return FP_ERR_ALIGNMENT;
  }
  if (p->head_bits && G > 8) return FP_ERR_UNSUPPORTED;  // one byte of head bits per list entry
  if (p->kv_lens) {  // chunked prefill reads the prefix from the paged cache
    if (!p->page_table || !p->cu_seqlens) return FP_ERR_INVALID_ARG;
    if (!aligned(p->kv_lens, 4)) return FP_ERR_ALIGNMENT;
  }
  if (p->page_table) {
    if (!p->cu_seqlens) return FP_ERR_INVALID_ARG;
    const int P = p->page_size;
    if (P < 16 || P > 65536 || (P & (P - 1)) != 0) return FP_ERR_UNSUPPORTED;
    if (p->num_pages < 1 || p->max_pages_per_req < ceil_div(p->max_seqlen, P)) return FP_ERR_INVALID_ARG;
  }
  if (attention) {
    int Tm = 1;
    while (Tm * 2 * G <= 128 && Tm * 2 <= p->block / 2) Tm *= 2;  // >= 2 M-tiles per query block
    if (p->block / Tm < 2) return FP_ERR_UNSUPPORTED;
  }
  return FP_OK;
}

Geometry geometry(const fp_params_t* p) {
  Geometry g;
  g.R = p->batch;
  g.L = p->max_seqlen;
  g.Hq = p->hq;
  g.Hkv = p->hkv;
  g.G = p->hq / p->hkv;
  g.d = p->head_dim;
  g.B = p->block;
  g.Nmax = ceil_div(g.L, g.B);
  g.Wmax = ceil_div(g.Nmax, 32);
  g.Sb = ceil_div(p->sink_tokens, g.B);
  g.Wb = ceil_div(p->window_tokens, g.B);
  if (g.Wb < 1) g.Wb = 1;
  g.scale = p->softmax_scale > 0.f ? p->softmax_scale : (float)(1.0 / std::sqrt((double)g.d));
  g.thr = p->alpha > 0.f ? (float)std::log((double)p->alpha) : -INFINITY;
  g.fp8 = p->dtype == FP_E4M3;
  g.cu = p->cu_seqlens;
  g.kv_lens = p->kv_lens;
  g.total_tokens = p->total_tokens;
  g.page_table = p->page_table;
  g.page_size = p->page_table ? p->page_size : 0;
  g.page_shift = 0;
  while (g.page_table && (1 << g.page_shift) < g.page_size) ++g.page_shift;
  g.max_pages = p->max_pages_per_req;
  g.num_pages = p->num_pages;
  g.q_scale = p->q_scale;
  g.k_scale = p->k_scale;
  g.v_scale = p->v_scale;
  g.head_bits = p->head_bits;
  g.status = nullptr;
  return g;
}

// Workspace: pooled query planes, pooled key planes (256-byte aligned), the
// attention work-queue counter (256 bytes), then the attention's claim order
// (one int per work unit; fp_prefill only).
size_t pad256(size_t bytes) { return (bytes + 255) / 256 * 256; }
size_t pooled_q_bytes(const Geometry& g) { return pad256(3 * pooled_q_elems(g) * sizeof(__nv_bfloat16)); }
size_t pooled_k_bytes(const Geometry& g) { return pad256(3 * pooled_k_elems(g) * sizeof(__nv_bfloat16)); }

int* queue_slot(const Geometry& g, void* ws) {
  return reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + pooled_q_bytes(g) + pooled_k_bytes(g));
}
int* order_slot(const Geometry& g, void* ws) { return queue_slot(g, ws) + 64; }

fp_status_t discover_impl(const fp_params_t* p, const void* q, const void* k, uint32_t* mask, int32_t* idx,
                          int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
  fp_status_t st = validate(p, false);
  if (st != FP_OK) return st;
  if (!q || !k || (!mask && !idx) || (idx && !cnt)) return FP_ERR_INVALID_ARG;
  if (p->head_bits && !idx) return FP_ERR_INVALID_ARG;  // head bits follow the compacted lists
  if (!aligned(q, 16) || !aligned(k, 16) || (mask && !aligned(mask, 4)) || (idx && !aligned(idx, 4)) ||
      (cnt && !aligned(cnt, 4)))
    return FP_ERR_ALIGNMENT;
  if (!ws || !aligned(ws, 256) || ws_bytes < fp_workspace_size(p)) return FP_ERR_WORKSPACE;
  Geometry g = geometry(p);
  g.status = status_ptr();
  if (!g.status) return cuda_fail("device status symbol", cudaGetLastError());
  __nv_bfloat16* qpl = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* kpl = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + pooled_q_bytes(g));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = launch_pool(g, q, k, qpl, kpl, s);
  if (e != cudaSuccess) return cuda_fail("pool launch", e);
  return launch_score(g, qpl, kpl, mask, idx, cnt, s);
}

fp_status_t attention_impl(const fp_params_t* p, bool paged, const void* q, const void* k, const void* v,
                           const int32_t* idx, const int32_t* cnt, void* o, float* lse, void* stream) {
  fp_status_t st = validate(p, true);
  if (st != FP_OK) return st;
  if (paged != (p->page_table != nullptr)) return FP_ERR_INVALID_ARG;
  if (!q || !k || !v || !idx || !cnt || !o) return FP_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(idx, 4) ||
      !aligned(cnt, 4) || (lse && !aligned(lse, 4)))
    return FP_ERR_ALIGNMENT;
  Geometry g = geometry(p);
  g.status = status_ptr();
  if (!g.status) return cuda_fail("device status symbol", cudaGetLastError());
  return launch_attention(g, q, k, v, idx, cnt, o, lse, static_cast<cudaStream_t>(stream), nullptr, nullptr, false);
}

}  // namespace
}  // namespace fp

using namespace fp;

extern "C" {

size_t fp_workspace_size(const fp_params_t* p) {
  if (validate(p, false) != FP_OK) return 0;
  const Geometry g = geometry(p);
  // + work-queue counter + claim order (when the attention supports this geometry)
  return pooled_q_bytes(g) + pooled_k_bytes(g) + 256 + pad256((size_t)attention_units(g) * sizeof(int));
}

size_t fp_mask_words(const fp_params_t* p) {
  if (validate(p, false) != FP_OK) return 0;
  const Geometry g = geometry(p);
  return (size_t)g.R * g.Hkv * g.Nmax * g.Wmax;
}

size_t fp_list_capacity(const fp_params_t* p) {
  if (validate(p, false) != FP_OK) return 0;
  const Geometry g = geometry(p);
  return (size_t)g.R * g.Hkv * ((size_t)g.Nmax * (g.Nmax + 1) / 2);
}

size_t fp_count_entries(const fp_params_t* p) {
  if (validate(p, false) != FP_OK) return 0;
  const Geometry g = geometry(p);
  return (size_t)g.R * g.Hkv * g.Nmax;
}

fp_status_t fp_discover(const fp_params_t* p, const void* q, const void* k, uint32_t* mask, void* workspace,
                        size_t ws_bytes, void* stream) {
  if (!mask) return FP_ERR_INVALID_ARG;
  return discover_impl(p, q, k, mask, nullptr, nullptr, workspace, ws_bytes, stream);
}

fp_status_t fp_discover_compact(const fp_params_t* p, const void* q, const void* k, uint32_t* mask, int32_t* idx,
                                int32_t* cnt, void* workspace, size_t ws_bytes, void* stream) {
  if (!idx || !cnt) return FP_ERR_INVALID_ARG;
  return discover_impl(p, q, k, mask, idx, cnt, workspace, ws_bytes, stream);
}

fp_status_t fp_compact(const fp_params_t* p, const uint32_t* mask, int32_t* idx, int32_t* cnt, void* stream) {
  fp_status_t st = validate(p, false);
  if (st != FP_OK) return st;
  if (!mask || !idx || !cnt) return FP_ERR_INVALID_ARG;
  if (p->head_bits) return FP_ERR_INVALID_ARG;  // the mask holds the group union only
  if (!aligned(mask, 4) || !aligned(idx, 4) || !aligned(cnt, 4)) return FP_ERR_ALIGNMENT;
  Geometry g = geometry(p);
  g.status = status_ptr();
  if (!g.status) return cuda_fail("device status symbol", cudaGetLastError());
  const cudaError_t e = launch_compact(g, mask, idx, cnt, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP_OK : cuda_fail("compact launch", e);
}

fp_status_t fp_sparse_prefill(const fp_params_t* p, const void* q, const void* k, const void* v, const int32_t* idx,
                              const int32_t* cnt, void* o, float* lse, void* stream) {
  return attention_impl(p, false, q, k, v, idx, cnt, o, lse, stream);
}

fp_status_t fp_paged_sparse_prefill(const fp_params_t* p, const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* idx, const int32_t* cnt, void* o, float* lse, void* stream) {
  return attention_impl(p, true, q, k_pool, v_pool, idx, cnt, o, lse, stream);
}

fp_status_t fp_prefill(const fp_params_t* p, const void* q, const void* k, const void* v, uint32_t* mask,
                       int32_t* idx, int32_t* cnt, void* o, float* lse, void* workspace, size_t ws_bytes,
                       void* stream) {
  fp_status_t st = validate(p, true);
  if (st != FP_OK) return st;
  if (!v || !o) return FP_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(o, 16) || (lse && !aligned(lse, 4))) return FP_ERR_ALIGNMENT;
  if (!idx || !cnt) return FP_ERR_INVALID_ARG;
  st = discover_impl(p, q, k, mask, idx, cnt, workspace, ws_bytes, stream);
  if (st != FP_OK) return st;
  Geometry g = geometry(p);
  g.status = status_ptr();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // longest lists first: the claim order of the attention's device queue
  const cudaError_t e = launch_unit_order(g, cnt, order_slot(g, workspace), queue_slot(g, workspace), s);
  if (e != cudaSuccess) return cuda_fail("unit order launch", e);
  return launch_attention(g, q, k, v, idx, cnt, o, lse, s, queue_slot(g, workspace), order_slot(g, workspace),
                          /*pdl=*/true);
}

fp_status_t fp_get_device_status(uint32_t* bits, void* stream) {
  unsigned* sp = status_ptr();
  if (!sp) return FP_ERR_CUDA;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("stream synchronize", e);
  unsigned v = 0;
  e = cudaMemcpy(&v, sp, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("status read", e);
  if (v && (e = cudaMemset(sp, 0, sizeof(unsigned))) != cudaSuccess) return cuda_fail("status clear", e);
  if (bits) *bits = v;
  return v ? FP_ERR_DEVICE : FP_OK;
}

const char* fp_last_error(void) { return t_last_error; }

const char* fp_status_string(fp_status_t s) {
  switch (s) {
    case FP_OK: return "FP_OK";
    case FP_ERR_INVALID_ARG: return "FP_ERR_INVALID_ARG";
    case FP_ERR_UNSUPPORTED: return "FP_ERR_UNSUPPORTED";
    case FP_ERR_ALIGNMENT: return "FP_ERR_ALIGNMENT";
    case FP_ERR_WORKSPACE: return "FP_ERR_WORKSPACE";
    case FP_ERR_CUDA: return "FP_ERR_CUDA";
    case FP_ERR_DEVICE: return "FP_ERR_DEVICE";
  }
  return "FP_ERR_UNKNOWN";
}

}  // extern "C"
