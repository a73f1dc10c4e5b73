// muon_noalloc.cu -- muon_step for callers that cannot allocate device memory.
//
// Some host programs may not call cudaMalloc (or any allocator) at the point
// where they run the optimizer: a runtime that fixes its whole device-memory
// budget at start-up and hands out nothing afterwards, or a plugin / callback
// running inside another framework that owns every allocation.  Such callers
// cannot provide the workspace muon_step needs.  muon_step_noalloc runs the
// same step with its scratch taken from one file-scope device array of fixed
// size instead; it allocates nothing.
//
// The array lives in this library's device image, so every GPU that loads
// the library holds it (MUON_NOALLOC_SCRATCH_BYTES) until the process exits.
// Host code cannot use the array's name as a device address; every call looks
// the address up with cudaGetSymbolAddress on the current device (cheap once
// the device code is loaded), so a device reset or another context on the
// device never sees a stale address.  The first call on a device, or after a
// reset, loads the device code: make it before any stream capture.  All calls
// on a device share the one array: calls that overlap on the GPU (different
// streams, no ordering between them) race on it, so order them (one stream,
// or events).  The array keeps the previous call's contents; the step itself
// clears what must start at zero (the status word) and overwrites the rest
// before reading it.  muon_noalloc_scratch hands out the array's address so
// that muon_query_status can read the status word of the last step.
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/muon_b200.h"

// Records the one-line reason muon_last_error() returns (muon_api.cu).
void muon_set_last_error(const char* msg);

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MUON_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current device's context.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

muon_status lookup_failed(cudaError_t e) {
  char msg[256];
  snprintf(msg, sizeof(msg), "muon_step_noalloc scratch: address lookup failed: %s", cudaGetErrorString(e));
  muon_set_last_error(msg);
  return MUON_ERR_CUDA;
}

}  // namespace

extern "C" muon_status muon_step_noalloc(float* const* params, const void* const* grads,
                                         float* const* momentum, const muon_group* groups,
                                         int n_groups, float lr, float beta, float wd,
                                         int ns_steps, const float* coeffs, uint32_t flags,
                                         muon_stream_t stream) {
  const size_t need = muon_workspace_min_size(groups, n_groups, flags);
  if (n_groups > 0 && need == 0) {
    // invalid groups: muon_step reports the exact reason without touching the GPU
    return muon_step(params, grads, momentum, groups, n_groups, lr, beta, wd, ns_steps, coeffs,
                     flags, nullptr, 0, stream);
  }
  if (need > MUON_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "muon_step_noalloc: the largest matrix needs %zu bytes of scratch, more than the "
             "%zu-byte built-in scratch (MUON_NOALLOC_SCRATCH_BYTES); use muon_step with a workspace",
             need, static_cast<size_t>(MUON_NOALLOC_SCRATCH_BYTES));
    muon_set_last_error(msg);
    return MUON_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  const cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) return lookup_failed(e);
  return muon_step(params, grads, momentum, groups, n_groups, lr, beta, wd, ns_steps, coeffs,
                   flags, ws, MUON_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" muon_status muon_noalloc_scratch(void** device_ptr, size_t* bytes) {
  if (!device_ptr) {
    muon_set_last_error("muon_noalloc_scratch: device_ptr is NULL");
    return MUON_ERR_INVALID_ARG;
  }
  void* ws = nullptr;
  const cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) return lookup_failed(e);
  *device_ptr = ws;
  if (bytes) *bytes = MUON_NOALLOC_SCRATCH_BYTES;
  return MUON_OK;
}
