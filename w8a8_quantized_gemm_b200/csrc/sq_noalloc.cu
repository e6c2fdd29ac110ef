// sq_smooth_quant_weight_noalloc: the smoothed weight quantization for callers that
// cannot allocate device memory, with its scratch in a static device array.
//
// Who needs it: code that runs inside a host program which owns the whole device-memory
// plan and hands its components only the tensors of the current call — for example a
// plugin of an inference engine or server, or a service that fixes its memory footprint
// at start-up and forbids later allocations. Such a caller has no way to provide the
// workspace that the per-tensor form of sq_smooth_quant_weight asks for (one global
// maximum), so this entry point keeps that scratch in the library itself.
#include "sq.h"
#include "sq_internal.h"

#include <cstdio>

namespace {

// The scratch: a file-scope device array. Every GPU that loads this library holds these
// bytes until the process exits. The per-tensor quantization keeps its running global
// absmax (one 32-bit word) here; the array is sized for that with room to spare.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device. In host code the array's name is
// only a host-side stand-in, so the address is looked up with the device current. The
// lookup is a host-side query and is repeated on every call: an address kept from an
// earlier call would point into freed memory after the program reset the device.
sq_status scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    char msg[256];
    snprintf(msg, sizeof msg, "sq_smooth_quant_weight_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    return static_cast<sq_status>(sq::record_error(SQ_ERR_CUDA, msg));
  }
  *out = p;
  return SQ_OK;
}

}  // namespace

extern "C" sq_status sq_smooth_quant_weight_noalloc(const void* W_bf16, int64_t N, int64_t K, int64_t ldw,
                                                     const float* s, sq_gran gran, int8_t* Wq, float* w_scale,
                                                     sq_stream_t stream) {
  const size_t need = (gran == SQ_PER_TENSOR) ? sq_workspace_size(SQ_OP_SMOOTH_QUANT_WEIGHT, 0, N, K) : 0;
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "sq_smooth_quant_weight_noalloc: this shape needs %zu bytes of scratch, the static scratch holds %zu",
             need, kNoAllocScratchBytes);
    return static_cast<sq_status>(sq::record_error(SQ_ERR_WORKSPACE, msg));
  }
  void* scratch = nullptr;
  sq_status st = scratch_address(&scratch);
  if (st != SQ_OK) return st;
  // Same validation, kernels and results as sq_smooth_quant_weight; the per-tensor path
  // resets the global maximum in the scratch before it accumulates into it.
  return sq_smooth_quant_weight(W_bf16, N, K, ldw, s, gran, Wq, w_scale, scratch, kNoAllocScratchBytes, stream);
}
