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
// (16 MiB). Every GPU that loads this library holds that array until the process exits. Every
// call, with the target device current, looks up the array's device address with
// cudaGetSymbolAddress (the host-side symbol is only a stand-in, not a device pointer). The
// lookup is not cached, so it follows the module instance of the current context: after a
// cudaDeviceReset, or from a non-primary context, it returns that context's copy of the array.
// The first call in a context may load the library's device module, so make it before any stream
// capture. The call then runs the ordinary mxattn_forward path with that address as its
// workspace; no cudaMalloc, cudaFree or other allocating routine is called.
//
// Limits: mxattn_forward's host-side checks see a workspace of kNoAllocScratchBytes, so a shape
// whose workspace (mxattn_forward_workspace_size) exceeds it is rejected with MXATTN_ERR_WORKSPACE,
// and every other rejected call gets the code mxattn_forward gives it, before anything is
// launched. All calls on a device share the one array and it keeps the last call's contents:
// mxattn_forward zeroes the status word at the start of every call and overwrites every other
// byte it reads, so no state leaks between calls, but calls whose kernels overlap on the GPU
// (different streams, no ordering) race on the array. Serialise them, e.g. by issuing them on one
// stream. A device-side wait timeout is recorded only in the shared array's status word, which no
// caller can read: `out` is then unspecified and the call still returned MXATTN_OK.
#include <cuda_runtime.h>

#include "../../include/mxattn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = MXATTN_NOALLOC_MAX_WORKSPACE;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the static scratch in the current context (looked up on every call).
mxattn_status scratch_for_current_context(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) return MXATTN_ERR_CUDA;
  *out = p;
  return MXATTN_OK;
}

}  // namespace

extern "C" mxattn_status mxattn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                                                int Hq, int Hkv, int N, int d, int causal, int scale_mode, int pnq,
                                                int out_dtype, void* stream) {
  void* scratch = nullptr;
  const mxattn_status s = scratch_for_current_context(&scratch);
  if (s != MXATTN_OK) return s;
  return mxattn_forward(q, k, v, out, B, Hq, Hkv, N, d, causal, scale_mode, pnq, out_dtype, scratch,
                        kNoAllocScratchBytes, stream);
}

extern "C" mxattn_status mxattn_check_status_noalloc(void* stream, unsigned int* detail) {
  void* scratch = nullptr;
  const mxattn_status s = scratch_for_current_context(&scratch);
  if (s != MXATTN_OK) return s;
  return mxattn_check_status(scratch, stream, detail);
}
