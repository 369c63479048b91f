// attn_splitkv_decode_static: the split-KV decode for callers that cannot
// allocate device memory.
//
// Some callers have no way to call cudaMalloc at the point where they need a
// decode: code running under a caching or arena allocator that owns all device
// memory, plugins that are handed only input and output buffers, or hosts that
// forbid allocation after start-up.  The regular entry point needs a caller
// workspace for the per-split partial results; this one keeps that scratch in
// a fixed-size array in device global memory defined in this file.  The array
// is part of the library's device image, so every GPU that loads the library
// holds it until the process exits.
//
// In host code the array's name is only a host-side stand-in, not a device
// address: its device address is looked up with cudaGetSymbolAddress, once per
// device, with that device current, on the first call made on the device.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "skv_internal.h"

namespace {

// Largest scratch a call may need: fp32 partial O and LSE of every split,
// B * Hq * Lq * (D + 1) * 4 bytes per split (each part 256-byte aligned).
constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_decode_scratch on the current device (looked up once).
int static_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return 0;
}

}  // namespace

extern "C" skv_status attn_splitkv_decode_static(const void* q, const void* k, const void* v, void* out, float* lse,
                                                 int B, int Hq, int Hkv, int Lq, int Lkv, int D, float scale,
                                                 skv_dtype dtype, const int32_t* kv_len, int num_splits,
                                                 skv_stream_t stream) {
  // The checks that decide the split count come first (sizes, dtype, head
  // dimension, scale), then the size refusal, so an unsupported or invalid
  // problem gets the same status as from attn_splitkv_decode and an oversized
  // one is refused before the scratch array is touched.  Pointer checks and
  // the launches are those of attn_splitkv_decode, called at the end.
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lkv < 0 || D < 1 || Hq % Hkv != 0) return SKV_ERR_INVALID_ARG;
  if (num_splits < 0 || num_splits > skv::kSplitMax) return SKV_ERR_INVALID_ARG;
  if (dtype != SKV_BF16 && dtype != SKV_FP16 && dtype != SKV_FP32) return SKV_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SKV_ERR_INVALID_ARG;
  if (dtype == SKV_FP32 || (D != 64 && D != 128 && D != 256)) return SKV_ERR_UNSUPPORTED;
  int splits = num_splits;
  if (splits == 0) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return skv::cuda_status(e);
    const skv_status s = attn_splitkv_plan(B, Hq, Hkv, Lq, Lkv, D, sms, 0, &splits, nullptr);
    if (s != SKV_OK) return s;
  }
  if (attn_splitkv_workspace(B, Hq, Lq, D, splits) > kStaticScratchBytes) return SKV_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const int e = static_scratch(&scratch);
  if (e != 0) return skv::cuda_status(e);
  // The regular entry point does the rest (validation, launches) with the
  // static array as its workspace; it allocates nothing either.
  return attn_splitkv_decode(q, k, v, out, lse, B, Hq, Hkv, Lq, Lkv, D, scale, dtype, kv_len, splits, scratch,
                             kStaticScratchBytes, stream);
}
