// Internal (non-ABI) definitions shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "flashprefill.h"

namespace fp {

// Validated, derived geometry of one call. Built on the host from fp_params_t.
struct Geometry {
  int R;          // requests (batch)
  int L;          // max_seqlen (contiguous: every request's length)
  int Hq, Hkv, G, d;
  int B;          // block size (tokens)
  int Nmax;       // ceil(L / B)
  int Wmax;       // ceil(Nmax / 32) mask words per row
  int Sb, Wb;     // sink / window in blocks
  float scale;    // softmax scale
  float thr;      // ln(alpha) (-inf for alpha == 0)
  int fp8;        // Q/K/V are e4m3
  const int32_t* cu;        // device cu_seqlens or nullptr
  const int32_t* kv_lens;   // device KV length per request (chunked prefill) or nullptr
  int total_tokens;
  const int32_t* page_table;  // device or nullptr
  int page_size, page_shift, max_pages, num_pages;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  uint8_t* head_bits;       // per-head selection bits per list entry, or nullptr
  unsigned* status;         // device status word
};

// Start token (row of the packed/contiguous layout) and length of request r.
// Invalid cu_seqlens make the request empty and set FP_DEV_BAD_SEQLENS.
__device__ __forceinline__ void request_span(const Geometry& g, int r, int& off, int& len) {
  if (g.cu == nullptr) {
    off = r * g.L;
    len = g.L;
    return;
  }
  const int a = __ldg(g.cu + r), b = __ldg(g.cu + r + 1);
  if (a < 0 || b < a || b - a > g.L || b > g.total_tokens) {
    atomicOr(g.status, FP_DEV_BAD_SEQLENS);
    off = 0;
    len = 0;
    return;
  }
  off = a;
  len = b - a;
}

// Query rows and KV length of request r. The queries are the request's last
// qlen tokens, at positions kvlen - qlen .. kvlen - 1 (kvlen == qlen unless
// kv_lens is given); query t of the request sits in row qoff + t - (kvlen - qlen).
// Inconsistent lengths make the request empty and set FP_DEV_BAD_SEQLENS.
__device__ __forceinline__ void request_spans(const Geometry& g, int r, int& qoff, int& qlen, int& kvlen) {
  request_span(g, r, qoff, qlen);
  kvlen = qlen;
  if (g.kv_lens != nullptr) {
    const int kl = __ldg(g.kv_lens + r);
    if (kl < qlen || kl > g.L) {
      atomicOr(g.status, FP_DEV_BAD_SEQLENS);
      qlen = 0;
      kvlen = 0;
      return;
    }
    kvlen = kl;
  }
}

__host__ __device__ __forceinline__ long long list_row_base(int r, int kvh, int i, int Hkv, int Nmax) {
  return ((long long)r * Hkv + kvh) * ((long long)Nmax * (Nmax + 1) / 2) + (long long)i * (i + 1) / 2;
}

__host__ __device__ __forceinline__ long long row_index(int r, int kvh, int i, int Hkv, int Nmax) {
  return ((long long)r * Hkv + kvh) * Nmax + i;
}

// Pooled tensors in the workspace, each as three bf16 planes (hi, mid, lo):
// queries [3][R * Nmax][Hq][128], keys [3][R * Hkv][Nmax][128]. Elements per plane:
size_t pooled_q_elems(const Geometry& g);
size_t pooled_k_elems(const Geometry& g);

// host launchers
cudaError_t launch_pool(const Geometry& g, const void* q, const void* k, __nv_bfloat16* qpl, __nv_bfloat16* kpl,
                        cudaStream_t s);
// Returns FP_OK, FP_ERR_UNSUPPORTED or FP_ERR_CUDA (with the failing step recorded).
fp_status_t launch_score(const Geometry& g, const __nv_bfloat16* qpl, const __nv_bfloat16* kpl, uint32_t* mask,
                         int32_t* idx, int32_t* cnt, cudaStream_t s);
cudaError_t launch_compact(const Geometry& g, const uint32_t* mask, int32_t* idx, int32_t* cnt,
                           cudaStream_t s);
// Returns FP_OK, FP_ERR_UNSUPPORTED or FP_ERR_CUDA.
// queue: zeroed device counter for claim-order scheduling, or nullptr (static
// stride); order: the units in claim order (launch_unit_order). pdl: launch as
// a programmatic dependent of the previous kernel.
fp_status_t launch_attention(const Geometry& g, const void* q, const void* k, const void* v,
                             const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                             cudaStream_t s, int* queue, const int* order, bool pdl);
// Attention work units of this geometry (0 when the attention does not support it).
long long attention_units(const Geometry& g);
// Writes the attention's longest-first claim order (attention_units(g) ints)
// from the list lengths and zeroes the queue counter.
cudaError_t launch_unit_order(const Geometry& g, const int32_t* cnt, int* order, int* queue, cudaStream_t s);

// cuTensorMapEncodeTiled (through the runtime's driver entry point) with
// 128-byte swizzle, 256-byte L2 promotion and zero fill outside the tensor.
// On failure records the step (fp_last_error) and returns false.
bool encode_tiled(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box);

// Records the failing step of the calling thread's last FP_ERR_CUDA (read by fp_last_error).
void set_last_error(const char* step, int code, const char* detail);

}  // namespace fp
