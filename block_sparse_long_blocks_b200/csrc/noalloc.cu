// Discovery + compaction for callers that cannot allocate device memory.
//
// fp_discover_compact needs a caller-provided workspace for the pooled Q and
// K. Some callers have no way to obtain one: a plugin running inside a host
// engine that owns every byte of device memory and exposes no allocator, or a
// latency-critical path that must not call cudaMalloc (it can synchronise the
// whole device). This file gives them fp_discover_compact_static, which takes
// its scratch from a fixed array in the library's device image instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its kStaticScratchBytes until the process exits. In host code
// its name is only a host-side stand-in, so its device address is resolved
// with cudaGetSymbolAddress, once per device, with that device current.
#include <cstdio>
#include <mutex>

#include "internal.cuh"

namespace fp {
namespace {

// 32 MiB: the pooled Q and K (three bf16 planes each) of one 128K-token
// sequence with 32 query and 4 KV heads at block 128 need 28.3 MB.
constexpr size_t kStaticScratchBytes = 32ull << 20;
constexpr int kMaxScratchDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (set up on the
// first call per device).
void* static_scratch_address() {
  static void* addr[kMaxScratchDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_error("cudaGetDevice", (int)e, cudaGetErrorString(e));
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxScratchDevices) {
    set_last_error("static scratch", dev, "device ordinal beyond the supported range");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) {
      set_last_error("cudaGetSymbolAddress(static scratch)", (int)e, cudaGetErrorString(e));
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace fp

extern "C" {

size_t fp_static_scratch_bytes(void) { return fp::kStaticScratchBytes; }

fp_status_t fp_discover_compact_static(const fp_params_t* p, const void* q, const void* k, uint32_t* mask,
                                       int32_t* idx, int32_t* cnt, void* stream) {
  const size_t need = fp_workspace_size(p);
  if (need == 0)  // invalid parameters: report the same status the workspace version would
    return fp_discover_compact(p, q, k, mask, idx, cnt, nullptr, 0, stream);
  if (need > fp::kStaticScratchBytes) {
    char msg[128];
    snprintf(msg, sizeof(msg), "needs %zu bytes of scratch, the static array holds %zu", need,
             fp::kStaticScratchBytes);
    fp::set_last_error("fp_discover_compact_static", 0, msg);
    return FP_ERR_WORKSPACE;
  }
  void* ws = fp::static_scratch_address();
  if (ws == nullptr) return FP_ERR_CUDA;
  return fp_discover_compact(p, q, k, mask, idx, cnt, ws, fp::kStaticScratchBytes, stream);
}

}  // extern "C"
