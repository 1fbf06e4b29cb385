// mxattn_forward_noalloc: MXFP4 attention forward for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host process whose device memory is owned by someone
// else -- an inference server or plugin host that hands out a fixed arena, a framework whose
// allocator must see every byte, or a latency-critical loop where an allocation call (which may
// synchronise the device or fail under a full memory pool) is not allowed. Such callers can pass
// inputs and outputs they already own, but cannot provide the workspace mxattn_forward needs for
// the quantized Q / K / V^T copies and the status word.
//
// How: the workspace lives in a file-scope static __device__ array of kNoAllocScratchBytes
// (16 MiB). Every GPU that loads this library holds that array until the process exits. The
// first call on a device, with that device current, looks up the array's device address with
// cudaGetSymbolAddress (the host-side symbol is only a stand-in, not a device pointer) and caches
// it per device; make that first call before any stream capture. Later calls reuse the address.
// The call then runs the ordinary mxattn_forward path with that address as its workspace; no
// cudaMalloc, cudaFree or other allocating routine is called.
//
// Limits: shapes whose workspace (mxattn_forward_workspace_size) exceeds kNoAllocScratchBytes are
// rejected with MXATTN_ERR_WORKSPACE before anything is launched. All calls on a device share the
// one array and it keeps the last call's contents: mxattn_forward zeroes the status word at the
// start of every call and overwrites every other byte it reads, so no state leaks between calls,
// but calls whose kernels overlap on the GPU (different streams, no ordering) race on the array.
// Serialise them, e.g. by issuing them on one stream.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mxattn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = MXATTN_NOALLOC_MAX_WORKSPACE;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device (looked up once per device).
mxattn_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MXATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return MXATTN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MXATTN_OK;
}

}  // namespace

extern "C" mxattn_status mxattn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                                                int Hq, int Hkv, int N, int d, int causal, int scale_mode, int pnq,
                                                int out_dtype, void* stream) {
  const size_t need = mxattn_forward_workspace_size(B, Hq, Hkv, N, d);
  if (need == 0) {
    // same argument classes as mxattn_forward for shapes it would reject
    if (d != 64 && d != 128 && B >= 1 && Hq >= 1 && Hkv >= 1 && N >= 1 && Hq % Hkv == 0)
      return MXATTN_ERR_UNSUPPORTED;
    return MXATTN_ERR_INVALID_ARG;
  }
  if (need > kNoAllocScratchBytes) return MXATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const mxattn_status s = scratch_for_current_device(&scratch);
  if (s != MXATTN_OK) return s;
  return mxattn_forward(q, k, v, out, B, Hq, Hkv, N, d, causal, scale_mode, pnq, out_dtype, scratch,
                        kNoAllocScratchBytes, stream);
}
